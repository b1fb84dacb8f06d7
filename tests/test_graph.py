"""A MoELayer step captured as one CUDA graph (MoEGraph, `MoELayer.capture`).

Replays on new tokens written into the static input equal the layer's eager
calls on the same tokens bit for bit (the same kernels on the same data, no
floating-point atomics on the forward path), and the first replay matches the
oracle: routing indices and plan bit-exact, outputs within the bf16 tolerance
(relative L2 1e-2)."""
import numpy as np
import pytest
import torch

from parity_util import BF16_TOL, check_outputs, check_routing, rel_l2, to_device
from sparse_mixture_experts_07_b200.inputs import MoEConfig, make_inputs, make_mxfp4_weights

pytestmark = pytest.mark.gpu

CASES = [
    MoEConfig("graph_decode_T1", T=1, H=512, I=256, E=16, k=2),
    MoEConfig("graph_decode_shared", T=8, H=256, I=128, E=8, k=2, n_shared=1, I_shared=128,
              routed_scale=2.5),
    MoEConfig("graph_T64", T=64, H=512, I=256, E=8, k=2, zipf_s=1.0),
    MoEConfig("graph_noaux", T=16, H=256, I=128, E=16, k=4, routing="noaux_tc", n_group=4,
              topk_group=2, zipf_s=1.2),
]
MX_CASES = [
    MoEConfig("graph_mx_T1", T=1, H=512, I=256, E=16, k=2),
    MoEConfig("graph_mx_T8", T=8, H=512, I=384, E=16, k=3, routed_scale=2.5),
    MoEConfig("graph_mx_T40", T=40, H=256, I=256, E=8, k=2),
]


def _layer(cfg, d, mx=None):
    import sparse_mixture_experts_07_b200 as moe
    shape = moe.Shape.from_config(cfg)
    routing = ("noaux_tc", cfg.n_group, cfg.topk_group) if cfg.routing == "noaux_tc" else None
    if mx is not None:
        return moe.MoELayer(shape, d["w_router"], d["router_bias"], mxfp4=mx, routing=routing)
    return moe.MoELayer(shape, d["w_router"], d["router_bias"], d["gate_up"], d["down"],
                        d["sh_gate_up"], d["sh_down"], routing=routing)


def _new_tokens(cfg, seed):
    g = torch.Generator().manual_seed(1000 + seed)
    return torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16).cuda()


def _replays_equal_eager(cfg, layer, graph, n=3):
    """Replay on n fresh token batches; each must equal an eager call bit for bit."""
    for seed in range(n):
        xn = _new_tokens(cfg, seed)
        graph.x.copy_(xn)
        y_graph = graph.replay().clone()
        idx_graph = layer.buf["topk_idx"].clone()
        torch.cuda.synchronize()
        y_eager = layer(xn).clone()
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        assert torch.equal(idx_graph, layer.buf["topk_idx"]), f"[{cfg.name}] routing differs"
        assert torch.equal(y_graph, y_eager), f"[{cfg.name}] replay {seed} differs from eager"


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_graph_bf16(cfg):
    import sparse_mixture_experts_07_b200 as moe
    inp = make_inputs(cfg, seed=0)
    d = to_device(inp)
    layer = _layer(cfg, d)
    x_static = torch.zeros_like(d["x"])
    graph = layer.capture(x_static)
    x_static.copy_(d["x"])
    y = graph.replay()
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    if cfg.routing == "softmax":
        shape = moe.Shape.from_config(cfg)
        _, _, logits = moe.route(shape, d["x"], d["w_router"], d["router_bias"], logits=True)
        res = {key: layer.buf[key].cpu() for key in ("topk_idx", "topk_w", "counts", "offsets",
                                                      "perm", "inv")}
        res["y"] = y.cpu()
        res["logits"] = logits.cpu()
        check_routing(cfg, inp, res)
        check_outputs(cfg, inp, res)
    else:
        # DeepSeek-V3 routing: the graph's first replay equals the eager call
        y0 = y.clone()
        torch.cuda.synchronize()
        assert torch.equal(layer(d["x"]), y0)
    _replays_equal_eager(cfg, layer, graph)


@pytest.mark.parametrize("cfg", MX_CASES, ids=lambda c: c.name)
def test_graph_mxfp4(cfg):
    from oracle import mxfp4
    inp = make_inputs(cfg, seed=0)
    mw = make_mxfp4_weights(cfg, seed=0)
    d = to_device(inp)
    layer = _layer(cfg, d, mx={key: v.cuda() for key, v in mw.items()})
    x_static = d["x"].clone()
    graph = layer.capture(x_static)
    y = graph.replay().cpu()
    assert layer.device_error() == 0
    y_o, idx_o, _ = mxfp4.moe_block_mxfp4(inp["x"], inp["w_router"], inp["router_bias"],
                                          mw["gate_up_q"], mw["gate_up_s"], mw["down_q"],
                                          mw["down_s"], k=cfg.k, routed_scale=cfg.routed_scale)
    assert np.array_equal(layer.buf["topk_idx"].cpu().numpy(), idx_o)
    err = rel_l2(y.float().numpy().astype(np.float64), y_o)
    print(f"[{cfg.name}] graph replay: mxfp4 rel L2 {err:.2e}")
    assert err <= BF16_TOL
    _replays_equal_eager(cfg, layer, graph)


def test_graph_rejects_wrong_shape():
    cfg = CASES[0]
    d = to_device(make_inputs(cfg, seed=0))
    layer = _layer(cfg, d)
    with pytest.raises(ValueError):
        layer.capture(torch.empty(cfg.T + 1, cfg.H, dtype=torch.bfloat16, device="cuda"))
