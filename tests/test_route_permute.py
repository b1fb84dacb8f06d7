"""moe_route_permute: the same outputs as moe_route_split followed by
moe_permute, bit for bit, whether it runs as one launch (up to 16 tokens on the
cluster router) or as the two calls; and the plan equals the oracle's on the
same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import to_device
from sparse_mixture_experts_07_b200.inputs import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    MoEConfig("rp_T1", T=1, H=512, I=64, E=16, k=2),
    MoEConfig("rp_T5_bias", T=5, H=1024, I=64, E=8, k=3, zipf_s=1.0),
    MoEConfig("rp_T16", T=16, H=2048, I=64, E=64, k=6, zipf_s=1.2),
    MoEConfig("rp_T16_k_equals_E", T=16, H=256, I=64, E=4, k=4),
    MoEConfig("rp_T9_E256_k8", T=9, H=2048, I=64, E=256, k=8),
    MoEConfig("rp_T3_f32", T=3, H=128, I=64, E=8, k=2, dtype="f32"),
    MoEConfig("rp_T17_two_calls", T=17, H=512, I=64, E=16, k=2),
    MoEConfig("rp_T300_tensor_core", T=300, H=512, I=64, E=16, k=2),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_route_permute_equals_the_two_calls(cfg):
    import sparse_mixture_experts_07_b200 as moe
    inp = make_inputs(cfg, seed=0)
    d = to_device(inp)
    shape = moe.Shape.from_config(cfg)
    ws = moe.alloc_workspace(shape)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    w_split = moe.router_split(shape, d["w_router"])
    fused = moe.route_permute(shape, d["x"], d["w_router"], d["router_bias"], ws, err,
                              logits=True, w_split=w_split)
    idx, w, lg = moe.route(shape, d["x"], d["w_router"], d["router_bias"], logits=True,
                           err_flag=err, w_split=w_split)
    plan = moe.permute(shape, idx, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for a, b, name in zip(fused, (idx, w, lg) + tuple(plan),
                          ("topk_idx", "topk_w", "logits", "counts", "offsets", "perm", "inv")):
        assert torch.equal(a, b), f"[{cfg.name}] {name} differs"
    # the plan against the oracle's (the generator keeps the top-k gaps, so
    # the oracle's selection is the same)
    o_idx, _ = oracle.topk_softmax(oracle.router(inp["x"], inp["w_router"], inp["router_bias"]),
                                   cfg.k)
    assert np.array_equal(fused[0].cpu().numpy(), o_idx)
    for got, want in zip(fused[3:], oracle.permute(o_idx, cfg.E)):
        assert np.array_equal(got.cpu().numpy(), want)


def _sweep_cases(n=24, seed=11):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        E = int(rng.choice([4, 8, 16, 32, 64, 128, 256]))
        k = int(rng.integers(1, min(E, 16) + 1))
        T = int(rng.integers(1, 17))
        H = int(rng.choice([8, 64, 200, 512, 1000, 2048]))
        cases.append((i, T, H, E, k, bool(rng.integers(0, 2))))
    return cases


@pytest.mark.parametrize("case", _sweep_cases(), ids=lambda c: f"sweep{c[0]}_T{c[1]}_H{c[2]}_E{c[3]}_k{c[4]}")
def test_route_permute_sweep_one_launch(case):
    """Random decode shapes on the one-launch path (T <= 16): routing and plan
    equal the two separate calls bit for bit (both run the same router, so
    near-ties resolve the same way), and the plan's invariants hold."""
    import sparse_mixture_experts_07_b200 as moe
    _, T, H, E, k, with_bias = case
    shape = moe.Shape(T=T, H=H, I=64, E=E, k=k)
    g = torch.Generator().manual_seed(T * 1000 + E * 10 + k)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16).cuda()
    wr = (torch.randn(E, H, generator=g) * 0.05).cuda()
    bias = (torch.randn(E, generator=g) * 0.5).cuda() if with_bias else None
    ws = moe.alloc_workspace(shape)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    fused = moe.route_permute(shape, x, wr, bias, ws, err, logits=True)
    idx, w, lg = moe.route(shape, x, wr, bias, logits=True, err_flag=err)
    plan = moe.permute(shape, idx, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for a, b in zip(fused, (idx, w, lg) + tuple(plan)):
        assert torch.equal(a, b)
    counts, offsets, perm, inv = (t.cpu().numpy() for t in fused[3:])
    sel = fused[0].cpu().numpy().reshape(-1)
    assert counts.sum() == T * k and offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(inv[perm], np.arange(T * k))
    keys = sel[perm].astype(np.int64) * (T * k) + perm
    assert np.all(np.diff(keys) > 0)
