"""The backward pass (moe_forward_train + moe_backward) against the oracle's
float64 gradients on the same seeded inputs and upstream gradient: every
gradient (x, both expert weights, router weight and bias, shared experts, the
routing weights) within relative L2 1e-2 (bf16 storage of the slot gradients
and pre-activations, float32 accumulation), the auxiliary loss's value and
gradient, and exact zeros for experts that received no token."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import rel_l2, to_device
from sparse_mixture_experts_07_b200.inputs import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-2

CONFIGS = [
    MoEConfig("bw_single", T=200, H=128, I=96, E=4, k=2),
    MoEConfig("bw_pair_shared", T=600, H=256, I=256, E=4, k=2, n_shared=1, I_shared=128,
              routed_scale=2.5, zipf_s=1.0),
    MoEConfig("bw_ragged", T=300, H=192, I=160, E=16, k=3, zipf_s=1.2),
    MoEConfig("bw_many_experts", T=256, H=256, I=128, E=64, k=6, n_shared=2, I_shared=64,
              routed_scale=2.5, zipf_s=1.2),
    MoEConfig("bw_empty_experts", T=20, H=128, I=64, E=16, k=1),
]


def _dy(cfg, seed=5):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16)


def _run(cfg, inp, dy, aux_coef=0.0):
    import sparse_mixture_experts_07_b200 as moe
    d = to_device(inp)
    shape = moe.Shape.from_config(cfg)
    # the layer only supplies buffers here: keep its shared experts as given
    layer = moe.MoELayer(shape, d["w_router"], d["router_bias"], d["gate_up"], d["down"],
                         d["sh_gate_up"], d["sh_down"], merge_shared=False)
    b = layer.buf
    idx, w, logits = moe.route(shape, d["x"], d["w_router"], d["router_bias"], out=b,
                               logits=True, err_flag=layer.err_flag, w_split=layer.w_split)
    moe.permute(shape, idx, layer.workspace, layer.err_flag, out=b)
    state = torch.empty(moe.train_state_size(shape), dtype=torch.uint8, device="cuda")
    moe.forward_train(shape, d["x"], b["offsets"], b["perm"], w, d["gate_up"], d["down"],
                      d["sh_gate_up"], d["sh_down"], layer.workspace, state, layer.err_flag,
                      y_slots=b["y_slots"])
    y = moe.combine(shape, b["y_slots"], b["inv"])
    ws = torch.empty(moe.backward_workspace_size(shape), dtype=torch.uint8, device="cuda")
    g = moe.backward(shape, d["x"], d["w_router"], idx, w, b["counts"], b["offsets"], b["perm"],
                     b["inv"], d["gate_up"], d["down"], d["sh_gate_up"], d["sh_down"], state,
                     dy.cuda(), ws, layer.err_flag, logits=logits, aux_coef=aux_coef,
                     want_topk_w_grad=True, want_aux_loss=True)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    out = {key: (v.cpu() if isinstance(v, torch.Tensor) else v) for key, v in g.items()}
    out["y"] = y.cpu()
    out["idx"] = idx.cpu()
    out["logits"] = logits.cpu()
    return out


def _cmp(name, got, want, tol=TOL):
    err = rel_l2(np.asarray(got, dtype=np.float64), want)
    print(f"  {name}: relative L2 {err:.2e}")
    assert err <= tol, f"{name}: relative L2 {err:.3e} > {tol}"


@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: c.name)
def test_backward_matches_oracle(cuda_ok, cfg):
    inp = make_inputs(cfg, seed=0)
    dy = _dy(cfg)
    res = _run(cfg, inp, dy)
    want = oracle.moe_backward(inp, cfg.k, dy.float().numpy(), routed_scale=cfg.routed_scale)
    print(f"[{cfg.name}]")
    for name in ("x", "gate_up", "down", "w_router", "router_bias"):
        _cmp(name, res[name].float().numpy(), want[name])
    if cfg.n_shared:
        _cmp("sh_gate_up", res["sh_gate_up"].numpy(), want["sh_gate_up"])
        _cmp("sh_down", res["sh_down"].numpy(), want["sh_down"])
    _cmp("topk_w", res["topk_w"].numpy(), want["dw"])
    # experts without tokens get exact zeros
    used = np.unique(res["idx"].numpy())
    for e in range(cfg.E):
        if e not in used:
            assert not res["gate_up"][e].any() and not res["down"][e].any()


def test_backward_aux_loss(cuda_ok):
    cfg = MoEConfig("bw_aux", T=300, H=128, I=64, E=8, k=2, zipf_s=1.0)
    inp = make_inputs(cfg, seed=0)
    dy = _dy(cfg, seed=6)
    coef = 0.01
    res = _run(cfg, inp, dy, aux_coef=coef)
    want = oracle.moe_backward(inp, cfg.k, dy.float().numpy(), routed_scale=cfg.routed_scale)
    lg = oracle.router(inp["x"], inp["w_router"], inp["router_bias"])
    idx, _ = oracle.topk_softmax(lg, cfg.k)
    loss, dl_aux = oracle.aux_loss(lg, idx, cfg.E, coef=coef)
    assert abs(float(res["aux_loss"][0]) - loss) <= 1e-5 * abs(loss) + 1e-7
    xf = inp["x"].float().numpy().astype(np.float64)
    wr = inp["w_router"].numpy().astype(np.float64)
    dl = want["dl"] + dl_aux
    _cmp("w_router (with aux)", res["w_router"].numpy(), dl.T @ xf)
    _cmp("router_bias (with aux)", res["router_bias"].numpy(), dl.sum(axis=0))
    _cmp("x (with aux)", res["x"].float().numpy(), want["x"] + dl_aux @ wr)


def test_backward_is_deterministic(cuda_ok):
    cfg = MoEConfig("bw_det", T=512, H=256, I=128, E=8, k=2, n_shared=1, I_shared=64)
    inp = make_inputs(cfg, seed=1)
    dy = _dy(cfg, seed=7)
    a = _run(cfg, inp, dy)
    b = _run(cfg, inp, dy)
    for key in ("x", "gate_up", "down", "sh_gate_up", "sh_down", "w_router", "router_bias"):
        assert torch.equal(a[key], b[key]), key
