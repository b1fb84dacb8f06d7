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
    """Worst-case bound on the router's float32 logit error (a ceiling only).

    The products x_h * w_h are exact on either router (bf16 x times the three
    bf16 terms of w, or float32 FMA).  The sum is float32: on the tensor cores
    the running sum is rounded once per 16-product MMA step, so H/16 roundings
    of at most 2^-23 of |logit| each; the CUDA-core router does fewer.  Twice
    that, plus 1e-6 for the weight split and the bias add."""
    return 2.0 * (H / 16.0) * 2.0 ** -23 * float(np.abs(logits).max()) + 1e-6


# Probabilistic per-logit bound, checked element by element:
#   |l_gpu - l| <= C_LOGIT * sqrt(n) * 2^-23 * (sum_h |x_h w_eh| + |b_e|)
# where n is the number of float32 roundings in the router's accumulation
# chain.  The products are exact (bf16 x times the bf16 terms of w, or float32
# FMA); each rounding is at most 2^-23 of the magnitudes summed so far, which
# sum_h |x_h w_eh| bounds; the roundings are independent and of either sign,
# so their sum grows like sqrt(n).  n per router path (router_chain_length):
#   tensor cores (bf16, T > 256, E <= 64): one rounding per 16-product MMA step,
#     n = H / 16;
#   one CTA per token (T <= 256): per-lane chains of H / 32, then a 5-level
#     warp tree, n = H / 32 + 5;
#   CUDA-core tiled router (float32 x, or E > 64): sequential FMA chains, n = H.
# C_LOGIT = 1.  Measured on a B200, the largest ratio of the error to this
# bound over every configuration of the GPU suite is 0.35 (gpt-oss- and
# DeepSeek-shaped layers, tensor cores; the Mixtral-shaped layer 0.31).
C_LOGIT = 1.0


def router_chain_length(cfg) -> float:
    """Float32 roundings in one logit's accumulation on the path moe_route /
    moe_route_split takes for this configuration."""
    if cfg.T <= 256:
        return cfg.H / 32.0 + 5.0
    if cfg.dtype == "bf16" and cfg.E <= 64:
        return cfg.H / 16.0
    return float(cfg.H)


def logit_scale(x, w_router, bias, n_chain: float) -> np.ndarray:
    """sqrt(n_chain) * 2^-23 * (sum_h |x_h w_eh| + |b_e|) for every (token, expert)."""
    xa = np.abs(x.float().numpy().astype(np.float64) if hasattr(x, "float") else np.asarray(x))
    wa = np.abs(w_router.float().numpy().astype(np.float64) if hasattr(w_router, "float")
                else np.asarray(w_router))
    s = xa @ wa.T
    if bias is not None:
        b = bias.float().numpy() if hasattr(bias, "float") else np.asarray(bias)
        s = s + np.abs(b.astype(np.float64))[None, :]
    return np.sqrt(n_chain) * 2.0 ** -23 * s


# Softmax over the selected k: |dw_i| <= w_i (|dl_i| + sum_j w_j |dl_j|) <= 2 max|dl|.


def to_device(inp: dict, dev="cuda") -> dict:
    out = {}
    for key, v in inp.items():
        out[key] = v.to(dev).contiguous() if isinstance(v, torch.Tensor) else v
    return out


def run_gpu(cfg: MoEConfig, dinp: dict, merge_shared: bool = True) -> dict:
    """Every step through the C ABI; returns host copies of all outputs.
    `merge_shared`: two or more shared experts run as one merged expert (the
    layer's default) or as separate groups."""
    shape = moe.Shape.from_config(cfg)
    layer = moe.MoELayer(shape, dinp["w_router"], dinp["router_bias"], dinp["gate_up"],
                         dinp["down"], dinp["sh_gate_up"], dinp["sh_down"],
                         merge_shared=merge_shared)
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
    """Indices and plan bit-exact; logits within the per-logit bound (and the
    worst-case ceiling); weights within twice the largest logit bound of
    their token.  Returns the oracle's (idx, counts, offsets, perm)."""
    T, k, E = cfg.T, cfg.k, cfg.E
    lg = oracle.router(inp["x"], inp["w_router"], inp["router_bias"], tokens=tokens)
    o_idx, o_w = oracle.topk_softmax(lg, k)
    g_idx = res["topk_idx"].numpy()
    g_w = res["topk_w"].numpy()
    sel = slice(None) if tokens is None else np.asarray(tokens)
    assert np.array_equal(g_idx[sel], o_idx), "routing indices differ"
    x_sel = inp["x"] if tokens is None else inp["x"][torch.as_tensor(np.asarray(tokens))]
    scale = logit_scale(x_sel, inp["w_router"], inp["router_bias"], router_chain_length(cfg))
    errs = [np.abs(res["logits"].numpy()[sel] - lg)]
    if "logits_split" in res:
        errs.append(np.abs(res["logits_split"].numpy()[sel] - lg))
    lerr = float(max(float(e.max()) for e in errs))
    ratio = float(max(float((e / scale).max()) for e in errs))
    ceiling = logit_tol(cfg.H, lg)
    assert lerr <= ceiling, f"logit error {lerr:.3e} > worst-case {ceiling:.3e}"
    werr_tok = np.abs(g_w[sel] - o_w).max(axis=1)
    wtol_tok = 2.0 * C_LOGIT * scale.max(axis=1) + 1e-7
    wratio = float((werr_tok / wtol_tok).max())
    assert ratio <= C_LOGIT, f"logit error {ratio:.3f} x the per-logit bound"
    assert wratio <= 1.0, f"routing weight error {wratio:.3f} x its bound"
    print(f"[{cfg.name}] logit error {lerr:.2e} = {ratio:.3f} x scale "
          f"(scale max {float(scale.max()):.2e}), weight error "
          f"{float(werr_tok.max()):.2e} = {wratio:.3f} x bound")
    _record(cfg.name, logit_err=lerr, logit_ratio=ratio, weight_err=float(werr_tok.max()),
            weight_ratio=wratio, scale_max=float(scale.max()))
    o_counts, o_offsets, o_perm, o_inv = oracle.permute(o_idx, E) if tokens is None else \
        (None, None, None, None)
    if tokens is None:
        assert np.array_equal(res["counts"].numpy(), o_counts)
        assert np.array_equal(res["offsets"].numpy(), o_offsets)
        assert np.array_equal(res["perm"].numpy(), o_perm)
        assert np.array_equal(res["inv"].numpy(), o_inv)
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
    return o_idx, o_counts, o_offsets, o_perm


def check_outputs(cfg: MoEConfig, inp: dict, res: dict, tokens=None):
    """Relative L2 error of y over the tokens, and of every token's row on its own."""
    y_o, idx_o, _ = oracle.moe_block(inp, k=cfg.k, routed_scale=cfg.routed_scale, tokens=tokens)
    y_g = res["y"].float().numpy()
    if tokens is not None:
        y_g = y_g[np.asarray(tokens)]
    y_g = y_g.astype(np.float64)
    err = rel_l2(y_g, y_o)
    row = np.linalg.norm(y_g - y_o, axis=1) / np.maximum(np.linalg.norm(y_o, axis=1), 1e-300)
    worst = int(np.argmax(row))
    tol = tolerance(cfg)
    assert err <= tol, f"relative L2 error {err:.3e} > {tol}"
    assert row[worst] <= tol, \
        f"row {worst if tokens is None else int(np.asarray(tokens)[worst])}: relative L2 " \
        f"error {row[worst]:.3e} > {tol}"
    n = y_o.shape[0]
    print(f"[{cfg.name}] output relative L2 error {err:.2e}, worst row {row[worst]:.2e} "
          f"over {n} tokens (bound {tol})")
    _record(cfg.name, out_err=err, out_row_err=float(row[worst]), out_tokens=n)
    return err


def rel_l2_rows(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-300)


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    if n >= T:
        return np.arange(T)
    t = rng.choice(T, size=n - 2, replace=False)
    return np.unique(np.concatenate([[0, T - 1], t]))


def stratified_tokens(o_idx: np.ndarray, offsets: np.ndarray, perm: np.ndarray, n_target: int,
                      tile: int = 128, per_expert: int = 2, seed: int = 0) -> np.ndarray:
    """Tokens to check at full size, chosen from the ORACLE's plan so that every
    routed expert's output rows are exercised:
      - the tokens of the first and last sorted row of each expert's last
        `tile`-row m-tile (the ragged tail, and the half tiles of the CTA-pair
        kernel, whose granularity is 128 rows as well);
      - `per_expert` further random tokens of each expert;
      - the first and last token, then random tokens up to n_target."""
    rng = np.random.default_rng(seed)
    T, k = o_idx.shape
    E = len(offsets) - 1
    pick = {0, T - 1}
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b <= a:
            continue
        last0 = a + ((b - 1 - a) // tile) * tile
        for p in (a, last0, b - 1):
            pick.add(int(perm[p]) // k)
        for p in rng.integers(a, b, size=per_expert):
            pick.add(int(perm[p]) // k)
    if len(pick) < n_target:
        rest = np.setdiff1d(np.arange(T), np.fromiter(pick, dtype=np.int64))
        extra = rng.choice(rest, size=min(len(rest), n_target - len(pick)), replace=False)
        pick.update(int(t) for t in extra)
    return np.array(sorted(pick), dtype=np.int64)


_RECORD = {}


def _record(name: str, **kw):
    """Collects the measured errors per configuration; written at session end
    when PARITY_RECORD names a file (see conftest)."""
    _RECORD.setdefault(name, {}).update(kw)


def records() -> dict:
    return _RECORD
