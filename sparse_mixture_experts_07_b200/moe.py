"""Python binding of include/moe.h (ctypes).

Argument marshalling only: every step of the block runs in libmoe.so's CUDA
kernels.  PyTorch provides device memory and the current stream.  If the
library has not been built, every call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, replace
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_BAD_INDEX", 6: "MOE_ERR_TIMEOUT"}
EXPORTS = ("moe_status_str", "moe_workspace_size", "moe_route", "moe_permute", "moe_forward",
           "moe_combine", "moe_router_split_size", "moe_router_split", "moe_route_split",
           "moe_forward_mxfp4", "moe_forward_experts", "moe_combine_experts", "moe_cast_f32",
           "moe_route_noaux_tc", "moe_train_state_size", "moe_forward_train",
           "moe_backward_workspace_size", "moe_backward", "moe_shared_merge")


class MoEShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("I_shared", ctypes.c_int32), ("routed_scale", ctypes.c_float),
                ("dtype", ctypes.c_int32)]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libmoe.so (raises if it is missing: build it with
    `python -m sparse_mixture_experts_07_b200.build`)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libmoe.so is not built ({path}); run "
                           "`python -m sparse_mixture_experts_07_b200.build`")
    lib = ctypes.CDLL(path)
    P, S = ctypes.c_void_p, ctypes.POINTER(MoEShape)
    lib.moe_status_str.argtypes = [ctypes.c_int]
    lib.moe_status_str.restype = ctypes.c_char_p
    lib.moe_workspace_size.argtypes = [S, ctypes.POINTER(ctypes.c_size_t)]
    lib.moe_route.argtypes = [S, P, P, P, P, P, P, P, P]
    lib.moe_permute.argtypes = [S, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.moe_route_permute.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                      ctypes.c_size_t, P]
    lib.moe_mxfp4_prepared_size.argtypes = [S, ctypes.POINTER(ctypes.c_size_t)]
    lib.moe_mxfp4_prepare.argtypes = [S, P, P, P, P, P, ctypes.c_size_t, P]
    lib.moe_forward_mxfp4_prepared.argtypes = [S, P, P, P, P, P, P, P, P, P, P,
                                               ctypes.c_size_t, P]
    lib.moe_forward.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.moe_combine.argtypes = [S, P, P, P, P]
    lib.moe_shared_merge.argtypes = [S, P, P, P, P, P]
    lib.moe_router_split_size.argtypes = [S, ctypes.POINTER(ctypes.c_size_t)]
    lib.moe_router_split.argtypes = [S, P, P, ctypes.c_size_t, P]
    lib.moe_route_split.argtypes = [S, P, P, P, P, P, P, P, P, P]
    lib.moe_forward_mxfp4.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    i32 = ctypes.c_int32
    lib.moe_forward_experts.argtypes = [S, i32, i32, P, P, P, P, P, P, P, P, P, P, P,
                                        ctypes.c_size_t, P]
    lib.moe_combine_experts.argtypes = [S, i32, i32, i32, P, P, P, P, P]
    lib.moe_cast_f32.argtypes = [S, P, P, P]
    lib.moe_route_noaux_tc.argtypes = [S, i32, i32, P, P, P, P, P, P, P, P, P]
    sz = ctypes.POINTER(ctypes.c_size_t)
    lib.moe_train_state_size.argtypes = [S, sz]
    lib.moe_forward_train.argtypes = [S, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P, P,
                                      ctypes.c_size_t, P]
    lib.moe_backward_workspace_size.argtypes = [S, sz]
    lib.moe_backward.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_float, P,
                                 P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    for f in EXPORTS[1:]:
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise MoEError(rc, where)


@dataclass(frozen=True)
class Shape:
    T: int
    H: int
    I: int
    E: int
    k: int
    n_shared: int = 0
    I_shared: int = 0
    routed_scale: float = 1.0
    dtype: int = MOE_BF16

    @staticmethod
    def from_config(cfg) -> "Shape":
        return Shape(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.n_shared, cfg.I_shared,
                     cfg.routed_scale, MOE_BF16 if cfg.dtype == "bf16" else MOE_F32)

    def c(self) -> MoEShape:
        return MoEShape(self.T, self.H, self.I, self.E, self.k, self.n_shared, self.I_shared,
                        self.routed_scale, self.dtype)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == MOE_BF16 else torch.float32

    @property
    def slot_rows(self) -> int:
        return self.T * (self.k + self.n_shared)


def workspace_size(shape: Shape) -> int:
    lib = load_library()
    n = ctypes.c_size_t(0)
    _check(lib.moe_workspace_size(ctypes.byref(shape.c()), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def alloc_workspace(shape: Shape, device="cuda") -> torch.Tensor:
    return torch.empty(max(workspace_size(shape), 1), dtype=torch.uint8, device=device)


def router_split(shape: Shape, w_router, stream=None):
    """The router weight split into three bf16 terms [N, H] (hi, mid, lo planes of
    E_PAD rows each, zero padding), for the tensor-core router; None when that
    router does not apply to `shape`.  Done once per weight."""
    lib = load_library()
    n = ctypes.c_size_t(0)
    _check(lib.moe_router_split_size(ctypes.byref(shape.c()), ctypes.byref(n)),
           "moe_router_split_size")
    if n.value == 0:
        return None
    ws = torch.empty(n.value // (2 * shape.H), shape.H, dtype=torch.bfloat16,
                     device=w_router.device)
    _check(lib.moe_router_split(ctypes.byref(shape.c()), _ptr(w_router), _ptr(ws), n.value,
                                _stream(stream)), "moe_router_split")
    return ws


def route(shape: Shape, x, w_router, router_bias=None, logits=False, out=None, stream=None,
          err_flag=None, w_split=None):
    """(topk_idx [T,k] int32, topk_w [T,k] f32, logits [T,E] f32 or None).
    `w_split` (from router_split) lets large batches skip the weight split."""
    lib = load_library()
    dev = x.device
    idx = out["topk_idx"] if out else torch.empty(shape.T, shape.k, dtype=torch.int32, device=dev)
    w = out["topk_w"] if out else torch.empty(shape.T, shape.k, dtype=torch.float32, device=dev)
    lg = torch.empty(shape.T, shape.E, dtype=torch.float32, device=dev) if logits else None
    if w_split is not None:
        _check(lib.moe_route_split(ctypes.byref(shape.c()), _ptr(x), _ptr(w_router),
                                   _ptr(w_split), _ptr(router_bias), _ptr(lg), _ptr(idx), _ptr(w),
                                   _ptr(err_flag), _stream(stream)), "moe_route_split")
    else:
        _check(lib.moe_route(ctypes.byref(shape.c()), _ptr(x), _ptr(w_router), _ptr(router_bias),
                             _ptr(lg), _ptr(idx), _ptr(w), _ptr(err_flag), _stream(stream)),
               "moe_route")
    return idx, w, lg


def route_noaux_tc(shape: Shape, x, w_router, score_bias, n_group: int, topk_group: int,
                   out=None, logits=None, stream=None, err_flag=None, w_split=None):
    """DeepSeek-V3 ("noaux_tc") routing: (topk_idx [T,k] int32, topk_w [T,k]
    f32, logits [T,E] f32).  `score_bias` steers the selection only."""
    lib = load_library()
    dev = x.device
    idx = out["topk_idx"] if out else torch.empty(shape.T, shape.k, dtype=torch.int32, device=dev)
    w = out["topk_w"] if out else torch.empty(shape.T, shape.k, dtype=torch.float32, device=dev)
    if logits is None:
        logits = torch.empty(shape.T, shape.E, dtype=torch.float32, device=dev)
    _check(lib.moe_route_noaux_tc(ctypes.byref(shape.c()), n_group, topk_group, _ptr(x),
                                  _ptr(w_router), _ptr(w_split), _ptr(score_bias), _ptr(logits),
                                  _ptr(idx), _ptr(w), _ptr(err_flag), _stream(stream)),
           "moe_route_noaux_tc")
    return idx, w, logits


def permute(shape: Shape, topk_idx, workspace, err_flag, out=None, stream=None):
    """(counts [E], offsets [E+1], perm [T*k], inv [T*k]) int32."""
    lib = load_library()
    dev = topk_idx.device
    n = shape.T * shape.k
    if out:
        counts, offsets, perm, inv = out["counts"], out["offsets"], out["perm"], out["inv"]
    else:
        counts = torch.empty(shape.E, dtype=torch.int32, device=dev)
        offsets = torch.empty(shape.E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(n, dtype=torch.int32, device=dev)
        inv = torch.empty(n, dtype=torch.int32, device=dev)
    _check(lib.moe_permute(ctypes.byref(shape.c()), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                           _ptr(perm), _ptr(inv), _ptr(err_flag), _ptr(workspace),
                           workspace.numel(), _stream(stream)), "moe_permute")
    return counts, offsets, perm, inv


def route_permute(shape: Shape, x, w_router, router_bias, workspace, err_flag, out=None,
                  logits=False, stream=None, w_split=None):
    """route then permute in one call (moe_route_permute; one launch for up to
    16 tokens): (topk_idx, topk_w, logits or None, counts, offsets, perm, inv)."""
    lib = load_library()
    dev = x.device
    n = shape.T * shape.k
    if out:
        idx, w = out["topk_idx"], out["topk_w"]
        counts, offsets, perm, inv = out["counts"], out["offsets"], out["perm"], out["inv"]
    else:
        idx = torch.empty(shape.T, shape.k, dtype=torch.int32, device=dev)
        w = torch.empty(shape.T, shape.k, dtype=torch.float32, device=dev)
        counts = torch.empty(shape.E, dtype=torch.int32, device=dev)
        offsets = torch.empty(shape.E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(n, dtype=torch.int32, device=dev)
        inv = torch.empty(n, dtype=torch.int32, device=dev)
    lg = torch.empty(shape.T, shape.E, dtype=torch.float32, device=dev) if logits else None
    _check(lib.moe_route_permute(ctypes.byref(shape.c()), _ptr(x), _ptr(w_router), _ptr(w_split),
                                 _ptr(router_bias), _ptr(lg), _ptr(idx), _ptr(w), _ptr(counts),
                                 _ptr(offsets), _ptr(perm), _ptr(inv), _ptr(err_flag),
                                 _ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_route_permute")
    return idx, w, lg, counts, offsets, perm, inv


def forward(shape: Shape, x, offsets, perm, topk_w, gate_up, down, sh_gate_up, sh_down,
            workspace, err_flag, y_slots=None, stream=None):
    """y_slots [T*k + S*T, H] (dtype): weighted expert outputs in sorted slot order,
    then the shared experts' outputs."""
    lib = load_library()
    if y_slots is None:
        y_slots = torch.empty(shape.slot_rows, shape.H, dtype=shape.torch_dtype, device=x.device)
    _check(lib.moe_forward(ctypes.byref(shape.c()), _ptr(x), _ptr(offsets), _ptr(perm),
                           _ptr(topk_w), _ptr(gate_up), _ptr(down), _ptr(sh_gate_up),
                           _ptr(sh_down), _ptr(y_slots), _ptr(err_flag), _ptr(workspace),
                           workspace.numel(), _stream(stream)), "moe_forward")
    return y_slots


def shared_merge(shape: Shape, sh_gate_up, sh_down, stream=None):
    """The shape's S shared experts as one of width S * I_shared (moe_shared_merge),
    done once at load time: (merged_shape, gate_up [1, 2 S Is, H], down [1, H, S Is])."""
    lib = load_library()
    S, Is, H = shape.n_shared, shape.I_shared, shape.H
    if sh_gate_up.shape != (S, 2 * Is, H) or sh_down.shape != (S, H, Is) \
            or not (sh_gate_up.is_contiguous() and sh_down.is_contiguous()):
        raise ValueError("shared experts must be contiguous [S, 2Is, H] and [S, H, Is]")
    gu = torch.empty(1, 2 * S * Is, H, dtype=shape.torch_dtype, device=sh_gate_up.device)
    dn = torch.empty(1, H, S * Is, dtype=shape.torch_dtype, device=sh_gate_up.device)
    _check(lib.moe_shared_merge(ctypes.byref(shape.c()), _ptr(sh_gate_up), _ptr(sh_down),
                                _ptr(gu), _ptr(dn), _stream(stream)), "moe_shared_merge")
    return replace(shape, n_shared=1, I_shared=S * Is), gu, dn


def forward_mxfp4(shape: Shape, x, offsets, perm, topk_w, mxfp4: dict, workspace, err_flag,
                  y_slots=None, stream=None):
    """moe_forward with MXFP4 routed-expert weights (decode batches, T <= 64):
    `mxfp4` holds gate_up_q, gate_up_s, down_q, down_s (uint8 device tensors)."""
    lib = load_library()
    if y_slots is None:
        y_slots = torch.empty(shape.slot_rows, shape.H, dtype=shape.torch_dtype, device=x.device)
    _check(lib.moe_forward_mxfp4(ctypes.byref(shape.c()), _ptr(x), _ptr(offsets), _ptr(perm),
                                 _ptr(topk_w), _ptr(mxfp4["gate_up_q"]), _ptr(mxfp4["gate_up_s"]),
                                 _ptr(mxfp4["down_q"]), _ptr(mxfp4["down_s"]), _ptr(y_slots),
                                 _ptr(err_flag), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "moe_forward_mxfp4")
    return y_slots


def mxfp4_prepare(shape: Shape, mxfp4: dict, stream=None):
    """`mxfp4` prepared once for the tensor-core kernel (moe_mxfp4_prepare: the
    scales in tensor-memory order, codes padded to whole 128-weight groups
    where H or I needs it): a uint8 device tensor, or None when the shape
    cannot take it (H or I not a multiple of 64)."""
    lib = load_library()
    n = ctypes.c_size_t(0)
    _check(lib.moe_mxfp4_prepared_size(ctypes.byref(shape.c()), ctypes.byref(n)),
           "moe_mxfp4_prepared_size")
    if n.value == 0:
        return None
    prepared = torch.empty(n.value, dtype=torch.uint8, device=mxfp4["gate_up_s"].device)
    _check(lib.moe_mxfp4_prepare(ctypes.byref(shape.c()), _ptr(mxfp4["gate_up_q"]),
                                 _ptr(mxfp4["gate_up_s"]), _ptr(mxfp4["down_q"]),
                                 _ptr(mxfp4["down_s"]), _ptr(prepared), n.value,
                                 _stream(stream)), "moe_mxfp4_prepare")
    return prepared


def forward_mxfp4_prepared(shape: Shape, x, offsets, perm, topk_w, mxfp4: dict, prepared,
                           workspace, err_flag, y_slots=None, stream=None):
    """moe_forward_mxfp4 on the tensor cores with the prepared weights (H and I
    multiples of 64): `mxfp4` supplies the raw gate_up_q and down_q."""
    lib = load_library()
    if y_slots is None:
        y_slots = torch.empty(shape.slot_rows, shape.H, dtype=shape.torch_dtype, device=x.device)
    _check(lib.moe_forward_mxfp4_prepared(ctypes.byref(shape.c()), _ptr(x), _ptr(offsets),
                                          _ptr(perm), _ptr(topk_w), _ptr(mxfp4["gate_up_q"]),
                                          _ptr(mxfp4["down_q"]), _ptr(prepared), _ptr(y_slots),
                                          _ptr(err_flag), _ptr(workspace), workspace.numel(),
                                          _stream(stream)), "moe_forward_mxfp4_prepared")
    return y_slots


def forward_experts(shape: Shape, e_begin: int, e_end: int, x, offsets, perm, topk_w,
                    gate_up_local, down_local, sh_gate_up, sh_down, workspace, err_flag,
                    y_slots, stream=None):
    """The expert FFNs of routed experts [e_begin, e_end) (their weights only),
    plus the shared experts when sh_gate_up / sh_down are given; writes those
    experts' rows of y_slots."""
    lib = load_library()
    _check(lib.moe_forward_experts(ctypes.byref(shape.c()), e_begin, e_end, _ptr(x),
                                   _ptr(offsets), _ptr(perm), _ptr(topk_w), _ptr(gate_up_local),
                                   _ptr(down_local), _ptr(sh_gate_up), _ptr(sh_down),
                                   _ptr(y_slots), _ptr(err_flag), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "moe_forward_experts")
    return y_slots


def combine_experts(shape: Shape, e_begin: int, e_end: int, with_shared: bool, y_slots, inv,
                    topk_idx, y_partial=None, stream=None):
    """float32 partial [T, H]: the slots of experts [e_begin, e_end) in token
    order (plus the shared experts' rows when with_shared)."""
    lib = load_library()
    if y_partial is None:
        y_partial = torch.empty(shape.T, shape.H, dtype=torch.float32, device=y_slots.device)
    _check(lib.moe_combine_experts(ctypes.byref(shape.c()), e_begin, e_end, int(with_shared),
                                   _ptr(y_slots), _ptr(inv), _ptr(topk_idx), _ptr(y_partial),
                                   _stream(stream)), "moe_combine_experts")
    return y_partial


def cast_f32(shape: Shape, y32, y=None, stream=None):
    """y [T, H] (dtype) = y32 rounded once."""
    lib = load_library()
    if y is None:
        y = torch.empty(shape.T, shape.H, dtype=shape.torch_dtype, device=y32.device)
    _check(lib.moe_cast_f32(ctypes.byref(shape.c()), _ptr(y32), _ptr(y), _stream(stream)),
           "moe_cast_f32")
    return y


def combine(shape: Shape, y_slots, inv, y=None, stream=None):
    """y [T, H] (dtype)."""
    lib = load_library()
    if y is None:
        y = torch.empty(shape.T, shape.H, dtype=shape.torch_dtype, device=y_slots.device)
    _check(lib.moe_combine(ctypes.byref(shape.c()), _ptr(y_slots), _ptr(inv), _ptr(y),
                           _stream(stream)), "moe_combine")
    return y


def train_state_size(shape: Shape) -> int:
    lib = load_library()
    n = ctypes.c_size_t(0)
    _check(lib.moe_train_state_size(ctypes.byref(shape.c()), ctypes.byref(n)),
           "moe_train_state_size")
    return n.value


def backward_workspace_size(shape: Shape) -> int:
    lib = load_library()
    n = ctypes.c_size_t(0)
    _check(lib.moe_backward_workspace_size(ctypes.byref(shape.c()), ctypes.byref(n)),
           "moe_backward_workspace_size")
    return n.value


def forward_train(shape: Shape, x, offsets, perm, topk_w, gate_up, down, sh_gate_up, sh_down,
                  workspace, state, err_flag, y_slots=None, stream=None):
    """moe_forward that also keeps, in `state`, what moe_backward reads."""
    lib = load_library()
    if y_slots is None:
        y_slots = torch.empty(shape.slot_rows, shape.H, dtype=shape.torch_dtype, device=x.device)
    _check(lib.moe_forward_train(ctypes.byref(shape.c()), _ptr(x), _ptr(offsets), _ptr(perm),
                                 _ptr(topk_w), _ptr(gate_up), _ptr(down), _ptr(sh_gate_up),
                                 _ptr(sh_down), _ptr(y_slots), _ptr(state), state.numel(),
                                 _ptr(err_flag), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "moe_forward_train")
    return y_slots


def backward(shape: Shape, x, w_router, topk_idx, topk_w, counts, offsets, perm, inv, gate_up,
             down, sh_gate_up, sh_down, state, dy, workspace, err_flag, logits=None,
             aux_coef: float = 0.0, want_topk_w_grad=False, want_aux_loss=False, stream=None):
    """The block's gradients: dict of dx (dtype), gate_up, down, sh_gate_up,
    sh_down, w_router, router_bias (float32), and topk_w / aux_loss if asked."""
    lib = load_library()
    dev = x.device
    f32 = torch.float32
    E, H, I, S = shape.E, shape.H, shape.I, shape.n_shared
    Is = shape.I_shared if S else 0
    g = {
        "x": torch.empty(shape.T, H, dtype=shape.torch_dtype, device=dev),
        "gate_up": torch.empty(E, 2 * I, H, dtype=f32, device=dev),
        "down": torch.empty(E, H, I, dtype=f32, device=dev),
        "sh_gate_up": torch.empty(S, 2 * Is, H, dtype=f32, device=dev) if S else None,
        "sh_down": torch.empty(S, H, Is, dtype=f32, device=dev) if S else None,
        "w_router": torch.empty(E, H, dtype=f32, device=dev),
        "router_bias": torch.empty(E, dtype=f32, device=dev),
        "topk_w": torch.empty(shape.T, shape.k, dtype=f32, device=dev) if want_topk_w_grad
        else None,
        "aux_loss": torch.zeros(1, dtype=f32, device=dev) if want_aux_loss else None,
    }
    _check(lib.moe_backward(ctypes.byref(shape.c()), _ptr(x), _ptr(w_router), _ptr(topk_idx),
                            _ptr(topk_w), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
                            _ptr(gate_up), _ptr(down), _ptr(sh_gate_up), _ptr(sh_down),
                            _ptr(state), _ptr(logits), float(aux_coef), _ptr(dy), _ptr(g["x"]),
                            _ptr(g["gate_up"]), _ptr(g["down"]), _ptr(g["sh_gate_up"]),
                            _ptr(g["sh_down"]), _ptr(g["w_router"]), _ptr(g["router_bias"]),
                            _ptr(g["topk_w"]), _ptr(g["aux_loss"]), _ptr(err_flag),
                            _ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_backward")
    return g


class MoELayer:
    """The whole block on one device: route -> permute -> forward -> combine.

    Holds the weights (device tensors) and a reusable workspace; `__call__`
    takes x [T, H] on the device and returns y [T, H].  Intermediates of the
    last call are kept in `self.last` for inspection.  Two or more shared
    experts are merged at construction into one of their summed width
    (moe_shared_merge): `self.shape` and `self.sh_gate_up` / `self.sh_down`
    are then the merged ones the library calls run on, and y_slots holds one
    shared row per token.
    """

    def __init__(self, shape: Shape, w_router, router_bias, gate_up=None, down=None,
                 sh_gate_up=None, sh_down=None, mxfp4=None, routing=None, merge_shared=True):
        """Expert weights either as gate_up / down (dtype of `shape`), or as
        `mxfp4` = {gate_up_q, gate_up_s, down_q, down_s} (decode batches).
        `routing`: None for top-k with a softmax over the selected k (the bias
        added to the logits), or ("noaux_tc", n_group, topk_group) for
        DeepSeek-V3 routing (the bias steers the selection only).
        `merge_shared`: run two or more shared experts as one (the default) or
        as separate groups."""
        self.shape = shape
        self.mxfp4 = mxfp4
        self.routing = routing
        if routing is not None and routing[0] != "noaux_tc":
            raise ValueError(f"unknown routing {routing!r}")
        self.w_router, self.router_bias = w_router, router_bias
        # split once here, at load time; refresh it if w_router changes
        self.w_split = router_split(shape, w_router)
        self.gate_up, self.down = gate_up, down
        self.sh_gate_up, self.sh_down = sh_gate_up, sh_down
        if merge_shared and shape.n_shared > 1 and mxfp4 is None:
            shape, self.sh_gate_up, self.sh_down = shared_merge(shape, sh_gate_up, sh_down)
            self.shape = shape
        # MXFP4 weights prepared once for the tensor-core kernel where it
        # takes the shape (decode batches, H and I multiples of 64)
        self.mx_prepared = None
        if (mxfp4 is not None and 1 <= shape.T <= 64 and shape.n_shared == 0
                and shape.dtype == MOE_BF16):
            self.mx_prepared = mxfp4_prepare(shape, mxfp4)
        dev = (gate_up if mxfp4 is None else mxfp4["gate_up_q"]).device
        self.workspace = alloc_workspace(shape, dev)
        self.err_flag = torch.zeros(1, dtype=torch.int32, device=dev)
        T, k, E, H = shape.T, shape.k, shape.E, shape.H
        self.buf = {
            "topk_idx": torch.empty(T, k, dtype=torch.int32, device=dev),
            "topk_w": torch.empty(T, k, dtype=torch.float32, device=dev),
            "counts": torch.empty(E, dtype=torch.int32, device=dev),
            "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "perm": torch.empty(T * k, dtype=torch.int32, device=dev),
            "inv": torch.empty(T * k, dtype=torch.int32, device=dev),
            "y_slots": torch.empty(shape.slot_rows, H, dtype=shape.torch_dtype, device=dev),
            "y": torch.empty(T, H, dtype=shape.torch_dtype, device=dev),
        }
        if routing is not None:
            self.buf["logits"] = torch.empty(T, E, dtype=torch.float32, device=dev)
        self.last = None

    def __call__(self, x, stream=None, y=None):
        s, b = self.shape, self.buf
        if self.routing is not None:
            idx, w, _ = route_noaux_tc(s, x, self.w_router, self.router_bias, self.routing[1],
                                       self.routing[2], out=b, logits=b["logits"],
                                       stream=stream, err_flag=self.err_flag,
                                       w_split=self.w_split)
            counts, offsets, perm, inv = permute(s, idx, self.workspace, self.err_flag, out=b,
                                                 stream=stream)
        else:
            idx, w, _, counts, offsets, perm, inv = route_permute(
                s, x, self.w_router, self.router_bias, self.workspace, self.err_flag, out=b,
                stream=stream, w_split=self.w_split)
        if self.mx_prepared is not None:
            forward_mxfp4_prepared(s, x, offsets, perm, w, self.mxfp4, self.mx_prepared,
                                   self.workspace, self.err_flag, y_slots=b["y_slots"],
                                   stream=stream)
        elif self.mxfp4 is not None:
            forward_mxfp4(s, x, offsets, perm, w, self.mxfp4, self.workspace, self.err_flag,
                          y_slots=b["y_slots"], stream=stream)
        else:
            forward(s, x, offsets, perm, w, self.gate_up, self.down, self.sh_gate_up,
                    self.sh_down, self.workspace, self.err_flag, y_slots=b["y_slots"],
                    stream=stream)
        out = combine(s, b["y_slots"], inv, y=b["y"] if y is None else y, stream=stream)
        self.last = b
        return out

    def device_error(self) -> int:
        """Device-detected error bits (synchronises)."""
        return int(self.err_flag.item())

    def capture(self, x, pool=None) -> "MoEGraph":
        """This layer's step on the static input `x` as a CUDA graph (MoEGraph)."""
        return MoEGraph(self, x, pool=pool)


class MoEGraph:
    """One MoELayer step (route, permute, forward, combine) captured once as a
    CUDA graph.

    Every launch of the step reads its shapes from the host and its routing
    from device buffers, so a graph replays the step exactly: write the next
    tokens into the static `x` (same shape, same storage) and call replay(),
    which leaves y [T, H] in `y` (the layer's output buffer).  Worth it for
    decode batches, where the step's launches cost about as much as streaming
    the active experts' weights.  The layer's buffers and workspace are shared
    with its eager calls; do not run both at once on different streams.
    """

    def __init__(self, layer: MoELayer, x, pool=None):
        if x.shape != (layer.shape.T, layer.shape.H):
            raise ValueError(f"x must be [{layer.shape.T}, {layer.shape.H}], got {tuple(x.shape)}")
        self.layer, self.x, self.y = layer, x, layer.buf["y"]
        dev = x.device
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            layer(x)  # first launches set kernel attributes outside the capture
        torch.cuda.current_stream(dev).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, pool=pool, stream=side):
            layer(x)

    def replay(self, stream=None):
        """Run the captured step on `stream` (default: the current stream); returns y."""
        if stream is None:
            self.graph.replay()
        else:
            with torch.cuda.stream(stream):
                self.graph.replay()
        return self.y
