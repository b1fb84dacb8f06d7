"""DeepSeek-V3 routing (noaux_tc) on the GPU against the oracle: bias-free
logits within the float32 bound, the selected experts bit-exact, their
weights within float32 rounding, the dispatch plan bit-exact, and the block's
outputs within the bf16 / float32 tolerance."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import (C_LOGIT, logit_scale, rel_l2, rel_l2_rows, router_chain_length,
                         stratified_tokens, to_device, tolerance)
from sparse_mixture_experts_07_b200.inputs import CONFIGS, MoEConfig, make_inputs

pytestmark = pytest.mark.gpu

SMALL = [
    MoEConfig("nx_dsv3_like", T=512, H=256, I=64, E=64, k=6, n_shared=2, I_shared=64,
              routed_scale=2.5, zipf_s=1.2, routing="noaux_tc", n_group=8, topk_group=4),
    MoEConfig("nx_groups_of_4", T=100, H=128, I=96, E=16, k=3, routing="noaux_tc", n_group=4,
              topk_group=2),
    MoEConfig("nx_one_group", T=300, H=200, I=64, E=32, k=4, zipf_s=1.0, routing="noaux_tc"),
    MoEConfig("nx_decode", T=5, H=256, I=128, E=16, k=2, routing="noaux_tc", n_group=4,
              topk_group=1),
    MoEConfig("nx_E256", T=700, H=128, I=64, E=256, k=8, routing="noaux_tc", n_group=32,
              topk_group=8),
    MoEConfig("nx_f32", T=64, H=96, I=64, E=8, k=2, dtype="f32", zipf_s=1.0,
              routing="noaux_tc", n_group=4, topk_group=2),
]


def _run(cfg, inp):
    import sparse_mixture_experts_07_b200 as moe
    d = to_device(inp)
    layer = moe.MoELayer(moe.Shape.from_config(cfg), d["w_router"], d["router_bias"],
                         d["gate_up"], d["down"], d["sh_gate_up"], d["sh_down"],
                         routing=("noaux_tc", cfg.n_group, cfg.topk_group))
    y = layer(d["x"])
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    return layer, y.cpu()


def _check(cfg, inp, layer, y, tokens=None):
    b = layer.last
    lg = oracle.router(inp["x"], inp["w_router"], None)
    o_idx, o_w = oracle.route_noaux_tc(lg, inp["router_bias"], cfg.k, cfg.n_group,
                                       cfg.topk_group)
    g_idx = b["topk_idx"].cpu().numpy()
    assert np.array_equal(g_idx, o_idx), "noaux_tc selection differs"
    # bias-free logits, element by element within the router's float32 bound
    scale = logit_scale(inp["x"], inp["w_router"], None, router_chain_length(cfg))
    lerr_el = np.abs(b["logits"].cpu().numpy() - lg)
    lerr = float(lerr_el.max())
    assert float((lerr_el / scale).max()) <= C_LOGIT, f"logit error {lerr:.3e}"
    # w = s_j / sum_i s_i with s = sigmoid(l): |ds| <= |dl| / 4, so each weight
    # moves by at most twice the token's largest logit error (plus rounding)
    werr = np.abs(b["topk_w"].cpu().numpy() - o_w).max(axis=1)
    wtol = 2.0 * C_LOGIT * scale.max(axis=1) + 1e-6
    assert (werr <= wtol).all(), f"weight error {float(werr.max()):.3e}"
    werr = float(werr.max())
    counts, offsets, perm, inv = oracle.permute(o_idx, cfg.E)
    assert np.array_equal(b["counts"].cpu().numpy(), counts)
    assert np.array_equal(b["perm"].cpu().numpy(), perm)
    assert np.array_equal(b["inv"].cpu().numpy(), inv)
    if tokens is None and cfg.T > 64:
        tokens = stratified_tokens(o_idx, offsets, perm, 256)
    y_o = oracle.moe_block_routed(inp, o_idx if tokens is None else o_idx[tokens],
                                  o_w if tokens is None else o_w[tokens],
                                  routed_scale=cfg.routed_scale, tokens=tokens)
    yg = y.float().numpy().astype(np.float64)
    if tokens is not None:
        yg = yg[tokens]
    err, rows = rel_l2(yg, y_o), rel_l2_rows(yg, y_o)
    print(f"[{cfg.name}] logit error {lerr:.2e}, weight error {werr:.2e}, output {err:.2e}, "
          f"worst row {rows.max():.2e}")
    assert err <= tolerance(cfg) and rows.max() <= tolerance(cfg)


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_noaux_small(cuda_ok, cfg):
    inp = make_inputs(cfg, seed=0)
    layer, y = _run(cfg, inp)
    _check(cfg, inp, layer, y)


def test_noaux_full_size_dsv3(cuda_ok):
    cfg = CONFIGS["dsv3_noaux"]
    inp = make_inputs(cfg, seed=0, weights_device="cuda")
    layer, y = _run(cfg, inp)
    host = {key: (v.cpu() if isinstance(v, torch.Tensor) else v) for key, v in inp.items()}
    lg = oracle.router(host["x"], host["w_router"], None)
    o_idx, _ = oracle.route_noaux_tc(lg, host["router_bias"], cfg.k, cfg.n_group,
                                     cfg.topk_group)
    _, offsets, perm, _ = oracle.permute(o_idx, cfg.E)
    toks = stratified_tokens(o_idx, offsets, perm, 1024)
    _check(cfg, host, layer, y, tokens=toks)
