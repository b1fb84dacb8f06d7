"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the CPU oracle on the same seeded inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_mixture_experts_07_b200 as moe
from sparse_mixture_experts_07_b200.inputs import MoEConfig, make_inputs

BF16_TOL = 1e-2     # relative L2 error bound for bf16 configurations
F32_TOL = 1e-5      # relative L2 error bound for float32 configurations


def logit_tol(H: int, logits: np.ndarray) -> float:
    """Bound on the router's float32 logit error.

    The products x_h * w_h are exact on either router (bf16 x times the three
    bf16 terms of w, or float32 FMA).  The sum is float32: on the tensor cores
    the running sum is rounded once per 16-product MMA step, so H/16 roundings
    of at most 2^-23 of |logit| each; the CUDA-core router does fewer.  Twice
    that, plus 1e-6 for the weight split and the bias add."""
    return 2.0 * (H / 16.0) * 2.0 ** -23 * float(np.abs(logits).max()) + 1e-6


# Softmax over the selected k: |dw_i| <= w_i (|dl_i| + sum_j w_j |dl_j|) <= 2 max|dl|.


def to_device(inp: dict, dev="cuda") -> dict:
    out = {}
    for key, v in inp.items():
        out[key] = v.to(dev).contiguous() if isinstance(v, torch.Tensor) else v
    return out


def run_gpu(cfg: MoEConfig, dinp: dict) -> dict:
    """Every step through the C ABI; returns host copies of all outputs."""
    shape = moe.Shape.from_config(cfg)
    layer = moe.MoELayer(shape, dinp["w_router"], dinp["router_bias"], dinp["gate_up"],
                         dinp["down"], dinp["sh_gate_up"], dinp["sh_down"])
    # logits of the router that splits the weight in every CTA, and of the
    # router on the weight split at load time (the layer's path)
    idx, w, logits = moe.route(shape, dinp["x"], dinp["w_router"], dinp["router_bias"],
                               logits=True)
    _, _, logits_split = moe.route(shape, dinp["x"], dinp["w_router"], dinp["router_bias"],
                                   logits=True, w_split=layer.w_split)
    y = layer(dinp["x"])
    torch.cuda.synchronize()
    b = layer.last
    res = {key: b[key].cpu() for key in ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv",
                                         "y_slots")}
    res["y"] = y.cpu()
    res["logits"] = logits.cpu()
    res["logits_split"] = logits_split.cpu()
    res["route_idx"] = idx.cpu()
    res["err"] = layer.device_error()
    return res


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def tolerance(cfg: MoEConfig) -> float:
    return BF16_TOL if cfg.dtype == "bf16" else F32_TOL


def check_routing(cfg: MoEConfig, inp: dict, res: dict, tokens=None):
    """Indices and plan bit-exact; weights within W_TOL; logits close."""
    T, k, E = cfg.T, cfg.k, cfg.E
    lg = oracle.router(inp["x"], inp["w_router"], inp["router_bias"], tokens=tokens)
    o_idx, o_w = oracle.topk_softmax(lg, k)
    g_idx = res["topk_idx"].numpy()
    g_w = res["topk_w"].numpy()
    sel = slice(None) if tokens is None else np.asarray(tokens)
    assert np.array_equal(g_idx[sel], o_idx), "routing indices differ"
    lerr = float(np.abs(res["logits"].numpy()[sel] - lg).max())
    if "logits_split" in res:
        lerr = max(lerr, float(np.abs(res["logits_split"].numpy()[sel] - lg).max()))
    werr = float(np.abs(g_w[sel] - o_w).max())
    ltol = logit_tol(cfg.H, lg)
    assert lerr <= ltol, f"logit error {lerr:.3e} > {ltol:.3e}"
    assert werr <= 2 * ltol, f"routing weight error {werr:.3e} > {2 * ltol:.3e}"
    print(f"[{cfg.name}] logit error {lerr:.2e} (bound {ltol:.2e}), weight error {werr:.2e}")
    if tokens is None:
        counts, offsets, perm, inv = oracle.permute(o_idx, E)
        assert np.array_equal(res["counts"].numpy(), counts)
        assert np.array_equal(res["offsets"].numpy(), offsets)
        assert np.array_equal(res["perm"].numpy(), perm)
        assert np.array_equal(res["inv"].numpy(), inv)
    else:
        # the plan's properties at any size
        counts = res["counts"].numpy()
        offsets = res["offsets"].numpy()
        perm = res["perm"].numpy()
        inv = res["inv"].numpy()
        assert counts.sum() == T * k
        assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
        assert np.array_equal(counts, np.bincount(g_idx.reshape(-1), minlength=E))
        assert np.array_equal(inv[perm], np.arange(T * k))
        keys = g_idx.reshape(-1)[perm].astype(np.int64) * (T * k) + perm
        assert np.all(np.diff(keys) > 0), "plan not ordered by (expert, slot)"


def check_outputs(cfg: MoEConfig, inp: dict, res: dict, tokens=None):
    y_o, idx_o, _ = oracle.moe_block(inp, k=cfg.k, routed_scale=cfg.routed_scale, tokens=tokens)
    y_g = res["y"].float().numpy()
    if tokens is not None:
        y_g = y_g[np.asarray(tokens)]
    err = rel_l2(y_g.astype(np.float64), y_o)
    assert err <= tolerance(cfg), f"relative L2 error {err:.3e} > {tolerance(cfg)}"
    print(f"[{cfg.name}] output relative L2 error {err:.2e} (bound {tolerance(cfg)})")
    return err


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    if n >= T:
        return np.arange(T)
    t = rng.choice(T, size=n - 2, replace=False)
    return np.unique(np.concatenate([[0, T - 1], t]))
