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


def test_mxfp4_weights_are_seeded_and_shaped():
    from sparse_mixture_experts_07_b200.inputs import MXFP4_SCALE_CODES, make_mxfp4_weights
    cfg = MoEConfig("mx", T=2, H=128, I=96, E=3, k=1)
    a = make_mxfp4_weights(cfg, seed=7)
    b = make_mxfp4_weights(cfg, seed=7)
    assert a["gate_up_q"].shape == (3, 192, 64) and a["gate_up_s"].shape == (3, 192, 4)
    assert a["down_q"].shape == (3, 128, 48) and a["down_s"].shape == (3, 128, 3)
    for key in a:
        assert a[key].dtype == torch.uint8 and torch.equal(a[key], b[key])
    scales = torch.cat([a["gate_up_s"].flatten(), a["down_s"].flatten()])
    assert set(scales.tolist()) <= set(MXFP4_SCALE_CODES)
    with pytest.raises(ValueError):
        make_mxfp4_weights(MoEConfig("bad", T=1, H=136, I=96, E=2, k=1))


def test_bench_rejects_mxfp4_outside_decode():
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--config", "mixtral",
                        "--weights", "mxfp4"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 2 and "decode configuration" in r.stderr


def test_decode_roofline_bytes():
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    cfg = CONFIGS["phimoe_decode1"]
    counts = np.zeros(cfg.E, dtype=np.int32)
    counts[[3, 9]] = 1
    act = 2 * cfg.T * cfg.H * 2 + 2 * cfg.T * cfg.k * cfg.H * 2 + cfg.E * cfg.H * 4
    assert bench.bytes_decode(cfg, counts) == 2 * 3 * cfg.H * cfg.I * 2 + act
    assert bench.bytes_decode(cfg, counts, mxfp4=True) == \
        2 * 3 * cfg.H * cfg.I * (0.5 + 1 / 32) + act


def test_noaux_inputs_have_clear_selection_gaps():
    """For DeepSeek-V3 routing the generator rejects near ties in the space the
    selection is taken in: sigmoid(logit) + bias, with group-limited top-k."""
    import oracle
    from sparse_mixture_experts_07_b200.inputs import GAP
    cfg = MoEConfig("nx_gen", T=400, H=128, I=64, E=32, k=4, zipf_s=1.0, routing="noaux_tc",
                    n_group=4, topk_group=2)
    inp = make_inputs(cfg, seed=3)
    lg = oracle.router(inp["x"], inp["w_router"], None)
    b = inp["router_bias"].numpy().astype(np.float64)
    c = 1.0 / (1.0 + np.exp(-lg)) + b
    gsize = cfg.E // cfg.n_group
    gs = np.sort(c.reshape(cfg.T, cfg.n_group, gsize), axis=2)[:, :, -2:].sum(axis=2)
    gsorted = -np.sort(-gs, axis=1)
    assert (gsorted[:, cfg.topk_group - 1] - gsorted[:, cfg.topk_group] > GAP).all()
    idx, _ = oracle.route_noaux_tc(lg, inp["router_bias"], cfg.k, cfg.n_group, cfg.topk_group)
    kept = np.argsort(-gs, axis=1)[:, :cfg.topk_group]
    for t in range(cfg.T):
        allowed = np.concatenate([np.arange(g * gsize, (g + 1) * gsize) for g in kept[t]])
        top = np.sort(c[t, allowed])[::-1][:cfg.k + 1]
        assert (np.diff(-top) > GAP).all()
        assert set(idx[t].tolist()) == set(allowed[np.argsort(-c[t, allowed])[:cfg.k]].tolist())
