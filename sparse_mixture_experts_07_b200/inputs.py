"""Seeded synthetic inputs for the dropless sparse MoE feed-forward block.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It draws random numbers and shapes them; it computes nothing
the MoE block computes for its result.  Two input-side checks do evaluate the
router's affine map in float64, only to choose inputs:

* near-tie rejection: a token row is redrawn until, on the exact stored values,
  its (k)-th and (k+1)-th largest router scores differ by more than 1e-3 and the
  k largest are pairwise more than 1e-3 apart, so that the expert selection and
  its order cannot depend on the rounding of either implementation (for
  DeepSeek-V3 routing the scores are sigmoid(logit) + bias, and the kept and
  first dropped group scores must be 1e-3 apart as well);
* Zipf load calibration: a per-expert router bias is fitted so that the share
  of tokens routed to expert e follows a Zipf law (the gpt-oss- and
  DeepSeek-V3-shaped workloads).

Neither implementation ever reads a number this module derives other than the
inputs themselves.

Shapes follow the models the pages describe:
  * PhiMoE (Phi-3.5-MoE): hidden 4096, expert intermediate 6400, 16 local
    experts, 2 per token, weights initialised N(0, 0.02) ("PhiMoE in
    Transformers", section 3, PhimoeConfig table).
  * gpt-oss-20b: 32 experts, 4 active per token ("Mixture of Experts in
    Transformers", section "from dense to sparse").
  * DeepSeek-V3-derived Instella-MoE: 64 routed + 2 shared experts, 6 per
    token, routed scale 2.5 (Instella-MoE modeling walk-through, "config at a
    glance").
  * Mixtral-8x7B: 8 experts, top-2 (PhiMoE is "very similar to Mixtral").
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

GAP = 1e-3          # minimum router-score gap around and inside the top-k
INIT_STD = 0.02     # initializer_range of the described configs


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                 # tokens
    H: int                 # hidden size
    I: int                 # expert intermediate size
    E: int                 # routed experts
    k: int                 # experts per token
    n_shared: int = 0      # always-on shared experts
    I_shared: int = 0      # shared expert intermediate size
    routed_scale: float = 1.0
    dtype: str = "bf16"    # activations and expert weights: "bf16" or "f32"
    zipf_s: Optional[float] = None   # None: unbiased router
    # "softmax": top-k of the (biased) logits, softmax over the k; "noaux_tc":
    # DeepSeek-V3 routing (sigmoid scores, bias in the selection only, the k
    # experts drawn from the topk_group best of n_group expert groups)
    routing: str = "softmax"
    n_group: int = 1
    topk_group: int = 1

    @property
    def slots(self) -> int:
        return self.T * self.k

    def flops(self) -> float:
        """Algorithmic flops of one layer: router + routed experts + shared experts."""
        T, H, I, E, k = self.T, self.H, self.I, self.E, self.k
        return 2.0 * T * (H * E + 3 * k * H * I + 3 * self.n_shared * self.I_shared * H)

    def with_tokens(self, T: int, name: Optional[str] = None) -> "MoEConfig":
        return dataclasses.replace(self, T=T, name=name or f"{self.name}_T{T}")


CONFIGS = {
    "tiny": MoEConfig("tiny", T=64, H=128, I=256, E=8, k=2, dtype="f32"),
    "mixtral": MoEConfig("mixtral", T=4096, H=4096, I=14336, E=8, k=2),
    "phimoe_prefill": MoEConfig("phimoe_prefill", T=8192, H=4096, I=6400, E=16, k=2),
    "phimoe_decode1": MoEConfig("phimoe_decode1", T=1, H=4096, I=6400, E=16, k=2),
    "phimoe_decode8": MoEConfig("phimoe_decode8", T=8, H=4096, I=6400, E=16, k=2),
    "phimoe_decode64": MoEConfig("phimoe_decode64", T=64, H=4096, I=6400, E=16, k=2),
    "gptoss": MoEConfig("gptoss", T=16384, H=2880, I=2880, E=32, k=4, zipf_s=1.0),
    # decode batches of the same layer (gpt-oss stores its experts in mxfp4)
    "gptoss_decode1": MoEConfig("gptoss_decode1", T=1, H=2880, I=2880, E=32, k=4, zipf_s=1.0),
    "gptoss_decode8": MoEConfig("gptoss_decode8", T=8, H=2880, I=2880, E=32, k=4, zipf_s=1.0),
    "dsv3": MoEConfig("dsv3", T=32768, H=2048, I=1024, E=64, k=6, n_shared=2,
                      I_shared=1024, routed_scale=2.5, zipf_s=1.2),
    # the same layer with the DeepSeek-V3 routing the Instella page names
    # (noaux_tc); 8 groups with 4 kept, DeepSeek-V3's published values
    "dsv3_noaux": MoEConfig("dsv3_noaux", T=32768, H=2048, I=1024, E=64, k=6, n_shared=2,
                            I_shared=1024, routed_scale=2.5, zipf_s=1.2, routing="noaux_tc",
                            n_group=8, topk_group=4),
}


def zipf_targets(E: int, k: int, s: float) -> np.ndarray:
    """Expected fraction of tokens that pick each expert under a Zipf(s) law.

    Expert e has Zipf rank e+1; the shares sum to k (k picks per token).  A token
    picks an expert at most once, so a share above 1 is capped at 1 and the
    excess is handed to the uncapped experts in proportion to their Zipf weight
    (water filling).  Without the cap, s=1.2 with E=64, k=6 would ask for 1.75.
    """
    p = 1.0 / np.arange(1, E + 1, dtype=np.float64) ** s
    q = k * p / p.sum()
    capped = np.zeros(E, dtype=bool)
    for _ in range(E):
        over = (q > 1.0) & ~capped
        if not over.any():
            break
        capped |= over
        free = k - capped.sum()
        q[capped] = 1.0
        q[~capped] = free * p[~capped] / p[~capped].sum()
    return q


def _scores64(x32: np.ndarray, wr: np.ndarray, b: Optional[np.ndarray]) -> np.ndarray:
    s = x32.astype(np.float64) @ wr.astype(np.float64).T
    if b is not None:
        s += b.astype(np.float64)[None, :]
    return s


def _bad_rows(scores: np.ndarray, k: int) -> np.ndarray:
    """Rows whose top-(k+1) sorted scores are not all more than GAP apart."""
    E = scores.shape[1]
    m = min(k + 1, E)
    top = -np.sort(-scores, axis=1)[:, :m]
    gaps = top[:, :-1] - top[:, 1:]
    if gaps.shape[1] == 0:
        return np.zeros(scores.shape[0], dtype=bool)
    return (gaps <= GAP).any(axis=1)


def _sigmoid64(v: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-v))


def _noaux_bad_rows(logits: np.ndarray, bias: Optional[np.ndarray], k: int, n_group: int,
                    topk_group: int) -> np.ndarray:
    """Rows whose noaux_tc decisions have a near tie (gap <= GAP): between the
    kept and the first dropped group score, or among the k + 1 largest
    selection scores of the kept groups."""
    T, E = logits.shape
    c = _sigmoid64(logits) + (0.0 if bias is None else bias.astype(np.float64)[None, :])
    gsize = E // n_group
    gs = np.sort(c.reshape(T, n_group, gsize), axis=2)[:, :, -min(2, gsize):].sum(axis=2)
    order = np.argsort(-gs, axis=1)
    gsorted = np.take_along_axis(gs, order, axis=1)
    bad = np.zeros(T, dtype=bool)
    if topk_group < n_group:
        bad |= gsorted[:, topk_group - 1] - gsorted[:, topk_group] <= GAP
    keep = np.zeros((T, n_group), dtype=bool)
    np.put_along_axis(keep, order[:, :topk_group], True, axis=1)
    allowed = np.repeat(keep, gsize, axis=1)
    cm = np.where(allowed, c, -np.inf)
    m = min(k + 1, topk_group * gsize)
    top = -np.sort(-cm, axis=1)[:, :m]
    if m > 1:
        bad |= (top[:, :-1] - top[:, 1:] <= GAP).any(axis=1)
    return bad


def _loads(scores: np.ndarray, k: int) -> np.ndarray:
    T, E = scores.shape
    sel = np.argpartition(-scores, k - 1, axis=1)[:, :k]
    return np.bincount(sel.ravel(), minlength=E) / T


def calibrate_bias(base_scores: np.ndarray, k: int, target: np.ndarray,
                   iters: int = 200) -> np.ndarray:
    """Fit a per-expert bias so that the realised loads approach `target`.

    Damped fixed point in float64: b <- b + eta (log q - log load), with eta
    starting at half the spread of the unbiased scores and shrinking by 0.7
    whenever the worst load error grows (the plain iteration oscillates when
    the bias is large compared with the score spread)."""
    T, E = base_scores.shape
    b = np.zeros(E, dtype=np.float64)
    eta = 0.5 * float(base_scores.std())
    prev = None
    for _ in range(iters):
        load = _loads(base_scores + b[None, :], k)
        b += eta * (np.log(target) - np.log(np.maximum(load, 0.5 / T)))
        b -= b.mean()
        worst = float(np.abs(load - target).max())
        if prev is not None and worst > prev:
            eta *= 0.7
        prev = worst
    return b


def _round(t: torch.Tensor, dtype: str) -> torch.Tensor:
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def torch_dtype(dtype: str) -> torch.dtype:
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def make_inputs(cfg: MoEConfig, seed: int = 0, weights_device: str = "cpu",
                max_redraw_rounds: int = 100) -> dict:
    """Draw x, router weight/bias and expert weights for one configuration.

    x ~ N(0,1) and every weight ~ N(0, 0.02).  x, the router weight Wr [E,H]
    (float32) and the bias are drawn on the CPU from one generator seeded with
    `seed`, in this order: x, Wr, then redraws of rejected x rows.  The expert
    weights are drawn from a second generator on `weights_device` (seed+1), in
    the order gate_up [E,2I,H], down [E,H,I], shared gate_up [S,2Is,H], shared
    down [S,H,Is]; drawing them on the GPU keeps multi-GB configurations quick.
    Activations and expert weights are rounded to bf16 for bf16 configurations;
    Wr and the bias stay float32.

    Returns a dict with torch tensors `x`, `w_router`, `router_bias` (or None),
    `gate_up`, `down`, `sh_gate_up`, `sh_down` (or None) and the bookkeeping
    `zipf_target`, `redrawn_rows`.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    T, H, E, k = cfg.T, cfg.H, cfg.E, cfg.k
    x = _round(torch.randn(T, H, generator=g), cfg.dtype)
    wr = torch.randn(E, H, generator=g) * INIT_STD
    wr_np = wr.numpy()

    noaux = cfg.routing == "noaux_tc"
    bias_np = None
    target = None
    if cfg.zipf_s is not None:
        target = zipf_targets(E, k, cfg.zipf_s)
        base = _scores64(x.float().numpy(), wr_np, None)
        # noaux_tc selects on sigmoid(logit) + bias (the fit ignores the groups)
        bias_np = calibrate_bias(_sigmoid64(base) if noaux else base, k, target)
        bias_np = bias_np.astype(np.float32)

    redrawn = 0
    for _ in range(max_redraw_rounds):
        if noaux:
            bad = _noaux_bad_rows(_scores64(x.float().numpy(), wr_np, None), bias_np, k,
                                  cfg.n_group, cfg.topk_group)
        else:
            bad = _bad_rows(_scores64(x.float().numpy(), wr_np, bias_np), k)
        nbad = int(bad.sum())
        if nbad == 0:
            break
        redrawn += nbad
        rows = torch.from_numpy(np.nonzero(bad)[0])
        x[rows] = _round(torch.randn(nbad, H, generator=g), cfg.dtype)
    else:
        raise RuntimeError("near-tie rejection did not converge")

    gw = torch.Generator(device=weights_device).manual_seed(seed + 1)
    wdt = torch_dtype(cfg.dtype)

    def draw(*shape):
        t = torch.empty(*shape, dtype=torch.float32, device=weights_device)
        t.normal_(0.0, INIT_STD, generator=gw)
        return t.to(wdt)

    I, S, Is = cfg.I, cfg.n_shared, cfg.I_shared
    gate_up = draw(E, 2 * I, H)
    down = draw(E, H, I)
    sh_gate_up = draw(S, 2 * Is, H) if S > 0 else None
    sh_down = draw(S, H, Is) if S > 0 else None
    return {
        "x": x,
        "w_router": wr,
        "router_bias": None if bias_np is None else torch.from_numpy(bias_np),
        "gate_up": gate_up,
        "down": down,
        "sh_gate_up": sh_gate_up,
        "sh_down": sh_down,
        "zipf_target": target,
        "redrawn_rows": redrawn,
    }


# MXFP4 scale codes drawn for synthetic expert weights: 2^-8 or 2^-7.  With
# codes uniform over the 16 E2M1 values (root mean square 2.93) the weights
# then have a root mean square of about 0.018, near the initializer_range
# (0.02) above.
MXFP4_SCALE_CODES = (119, 120)


def make_mxfp4_weights(cfg: MoEConfig, seed: int = 0, device: str = "cpu") -> dict:
    """Routed expert weights in the MXFP4 storage layout, drawn at random.

    gate_up_q [E, 2I, H/2] and down_q [E, H, I/2] are uniform random bytes (two
    4-bit codes each); gate_up_s [E, 2I, H/32] and down_s [E, H, I/32] are drawn
    uniformly from MXFP4_SCALE_CODES.  One generator on `device` seeded with
    `seed` + 2, in that order.  H and I must be multiples of 32."""
    E, H, I = cfg.E, cfg.H, cfg.I
    if H % 32 or I % 32:
        raise ValueError("MXFP4 weights need H and I to be multiples of 32")
    g = torch.Generator(device=device).manual_seed(seed + 2)
    codes = torch.tensor(MXFP4_SCALE_CODES, dtype=torch.uint8, device=device)

    def qbytes(*shape):
        return torch.randint(0, 256, shape, generator=g, dtype=torch.uint8, device=device)

    def scales(*shape):
        return codes[torch.randint(0, len(MXFP4_SCALE_CODES), shape, generator=g,
                                   device=device)]

    return {
        "gate_up_q": qbytes(E, 2 * I, H // 2),
        "gate_up_s": scales(E, 2 * I, H // 32),
        "down_q": qbytes(E, H, I // 2),
        "down_s": scales(E, H, I // 32),
    }
