"""Decode steps back to back on alternating token batches.

The decode chain's kernels start as programmatic dependents of the kernel
before them and wait for it before touching memory that an earlier kernel
writes or reads.  Steps are issued back to back on one stream, with
different tokens each time and no other kernel in between (each step writes
its own output buffer); every output must equal the layer's output for those
tokens computed on their own, bit for bit (the same kernels on the same
data).  A kernel that read a buffer before the kernel writing it had
finished, or overwrote one still being read, would show as a mismatch."""
import pytest
import torch

from parity_util import to_device
from sparse_mixture_experts_07_b200.inputs import MoEConfig, make_inputs, make_mxfp4_weights

pytestmark = pytest.mark.gpu

CASES = [
    (MoEConfig("chain_bf16_T1", T=1, H=1024, I=512, E=16, k=2), "bf16"),
    (MoEConfig("chain_bf16_T8", T=8, H=2048, I=1024, E=16, k=2, zipf_s=1.0), "bf16"),
    (MoEConfig("chain_bf16_T8_shared", T=8, H=1024, I=512, E=8, k=2, n_shared=1, I_shared=256,
               routed_scale=2.5), "bf16"),
    (MoEConfig("chain_bf16_T64", T=64, H=1024, I=512, E=8, k=2), "bf16"),
    (MoEConfig("chain_mx_T1", T=1, H=1024, I=512, E=16, k=2), "mxfp4"),
    (MoEConfig("chain_mx_T8", T=8, H=2048, I=1024, E=16, k=3), "mxfp4"),
    (MoEConfig("chain_mx_T40", T=40, H=1024, I=512, E=8, k=2), "mxfp4"),
]


@pytest.mark.parametrize("cfg,weights", CASES, ids=lambda c: getattr(c, "name", c))
def test_back_to_back_steps(cfg, weights):
    import sparse_mixture_experts_07_b200 as moe
    d = to_device(make_inputs(cfg, seed=0))
    shape = moe.Shape.from_config(cfg)
    if weights == "mxfp4":
        mx = {key: v.cuda() for key, v in make_mxfp4_weights(cfg, seed=0).items()}
        layer = moe.MoELayer(shape, d["w_router"], d["router_bias"], mxfp4=mx)
    else:
        layer = moe.MoELayer(shape, d["w_router"], d["router_bias"], d["gate_up"], d["down"],
                             d["sh_gate_up"], d["sh_down"])
    g = torch.Generator().manual_seed(7)
    xs = [torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16).cuda() for _ in range(3)]
    refs = []
    for x in xs:
        refs.append(layer(x).clone())
        torch.cuda.synchronize()
    assert layer.device_error() == 0
    rounds = 6
    outs = [torch.empty_like(refs[0]) for _ in range(rounds * len(xs))]
    torch.cuda.synchronize()
    for r in range(rounds):
        for i, x in enumerate(xs):
            layer(x, y=outs[r * len(xs) + i])
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    for n, y in enumerate(outs):
        assert torch.equal(y, refs[n % len(xs)]), f"[{cfg.name}] step {n} differs"
