"""The seeded input generator: gaps, Zipf targets, determinism."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_07_b200.inputs import (CONFIGS, GAP, MoEConfig, make_inputs,
                                                   zipf_targets)


def _sorted_scores(inp):
    s = inp["x"].double() @ inp["w_router"].double().T
    if inp["router_bias"] is not None:
        s = s + inp["router_bias"].double()[None]
    return torch.sort(s, dim=1, descending=True).values


@pytest.mark.parametrize("name", ["tiny", "phimoe_decode64"])
def test_gap_guarantee(name):
    cfg = CONFIGS[name]
    inp = make_inputs(cfg)
    top = _sorted_scores(inp)[:, :cfg.k + 1]
    assert bool(((top[:, :-1] - top[:, 1:]) > GAP).all())


def test_generator_is_deterministic():
    a = make_inputs(CONFIGS["tiny"], seed=3)
    b = make_inputs(CONFIGS["tiny"], seed=3)
    for key in ("x", "w_router", "gate_up", "down"):
        assert torch.equal(a[key], b[key])
    c = make_inputs(CONFIGS["tiny"], seed=4)
    assert not torch.equal(a["x"], c["x"])


def test_distributions():
    cfg = MoEConfig("t", T=256, H=256, I=128, E=8, k=2, dtype="bf16")
    inp = make_inputs(cfg)
    assert inp["x"].dtype == torch.bfloat16 and inp["w_router"].dtype == torch.float32
    assert abs(inp["x"].float().std().item() - 1.0) < 0.02
    assert abs(inp["gate_up"].float().std().item() - 0.02) < 0.001
    assert inp["gate_up"].shape == (8, 256, 256) and inp["down"].shape == (8, 256, 128)


@pytest.mark.parametrize("E,k,s", [(32, 4, 1.0), (64, 6, 1.2), (8, 2, 0.5)])
def test_zipf_targets_feasible(E, k, s):
    q = zipf_targets(E, k, s)
    assert abs(q.sum() - k) < 1e-12
    assert np.all(q <= 1.0 + 1e-12) and np.all(q > 0)
    assert np.all(np.diff(q) <= 1e-12)


def test_zipf_calibration_reaches_target():
    cfg = MoEConfig("z", T=4096, H=256, I=64, E=16, k=4, zipf_s=1.0)
    inp = make_inputs(cfg)
    s = inp["x"].double() @ inp["w_router"].double().T + inp["router_bias"].double()[None]
    sel = torch.topk(s, cfg.k, dim=1).indices
    load = torch.bincount(sel.reshape(-1), minlength=cfg.E).double() / cfg.T
    q = torch.from_numpy(inp["zipf_target"])
    assert float((load - q).abs().max()) < 0.03
