"""MXFP4 expert weights on the decode path (moe_forward_mxfp4, 1 <= T <= 64)
against the oracle's MXFP4 block, on the same seeded inputs: routing bit-exact,
outputs within the bf16 tolerance (relative L2 1e-2), over the batch and row
by row."""
import numpy as np
import pytest
import torch

from parity_util import BF16_TOL, rel_l2, rel_l2_rows, to_device
from sparse_mixture_experts_07_b200.inputs import CONFIGS, MoEConfig, make_inputs, make_mxfp4_weights

pytestmark = pytest.mark.gpu

SMALL = [
    MoEConfig("mx_one_token", T=1, H=256, I=128, E=8, k=2),
    MoEConfig("mx_ragged", T=7, H=512, I=320, E=16, k=3, routed_scale=2.5),
    MoEConfig("mx_k_equals_E", T=8, H=128, I=64, E=4, k=4),
    MoEConfig("mx_odd_blocks", T=5, H=288, I=96, E=6, k=2, zipf_s=1.0),
    # 9..64 tokens: chunks of up to 32 rows per expert group (four 8-token tiles)
    MoEConfig("mx_T9", T=9, H=256, I=128, E=8, k=2),
    MoEConfig("mx_T40_ragged", T=40, H=544, I=224, E=8, k=3, routed_scale=2.5),
    # a group of more than 32 rows runs as several chunks
    MoEConfig("mx_T64_two_chunks", T=64, H=256, I=192, E=4, k=2, zipf_s=1.2),
    MoEConfig("mx_T64_odd_blocks", T=64, H=288, I=160, E=16, k=4, zipf_s=1.0),
    # H and I multiples of 128: the block-scaled tensor-core kernel, chunks of
    # 8 (T <= 8) and 16 rows (several per expert at T = 33 and 64),
    # contraction splits for small batches
    MoEConfig("mx_tc_ragged", T=7, H=512, I=384, E=16, k=3, routed_scale=2.5),
    MoEConfig("mx_tc_k_equals_E", T=8, H=128, I=128, E=4, k=4),
    MoEConfig("mx_tc_T16", T=16, H=384, I=256, E=8, k=2, zipf_s=1.0),
    MoEConfig("mx_tc_T64_two_chunks", T=64, H=256, I=256, E=4, k=2, zipf_s=1.2),
    MoEConfig("mx_tc_splits", T=1, H=2176, I=1152, E=8, k=2),
    MoEConfig("mx_tc_T33_splits", T=33, H=1024, I=512, E=32, k=2, zipf_s=1.0),
]


def _run(cfg, inp, mw):
    import sparse_mixture_experts_07_b200 as moe
    shape = moe.Shape.from_config(cfg)
    d = to_device(inp)
    dm = {key: v.cuda() for key, v in mw.items()}
    layer = moe.MoELayer(shape, d["w_router"], d["router_bias"], mxfp4=dm)
    y = layer(d["x"])
    torch.cuda.synchronize()
    return layer, y.cpu()


def _check(cfg, inp, mw, layer, y, tokens=None):
    from oracle import mxfp4
    y_o, idx_o, _ = mxfp4.moe_block_mxfp4(inp["x"], inp["w_router"], inp["router_bias"],
                                          mw["gate_up_q"], mw["gate_up_s"], mw["down_q"],
                                          mw["down_s"], k=cfg.k, routed_scale=cfg.routed_scale,
                                          tokens=tokens)
    sel = slice(None) if tokens is None else np.asarray(tokens)
    assert layer.device_error() == 0
    assert np.array_equal(layer.last["topk_idx"].cpu().numpy()[sel], idx_o)
    yg = y.float().numpy()[sel].astype(np.float64)
    err = rel_l2(yg, y_o)
    rows = rel_l2_rows(yg, y_o)
    print(f"[{cfg.name}] mxfp4 rel L2 {err:.2e}, worst row {rows.max():.2e}")
    assert err <= BF16_TOL
    assert rows.max() <= BF16_TOL


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_mxfp4_decode_small(cuda_ok, cfg):
    inp = make_inputs(cfg)
    mw = make_mxfp4_weights(cfg)
    layer, y = _run(cfg, inp, mw)
    _check(cfg, inp, mw, layer, y)


@pytest.mark.parametrize("name", ["phimoe_decode1", "phimoe_decode8", "phimoe_decode64"])
def test_mxfp4_decode_full_size(cuda_ok, name):
    cfg = CONFIGS[name]
    inp = make_inputs(cfg)
    mw = make_mxfp4_weights(cfg)
    layer, y = _run(cfg, inp, mw)
    _check(cfg, inp, mw, layer, y)


def test_mxfp4_slot_rows_hold_weighted_expert_outputs(cuda_ok):
    from oracle import expert
    from oracle.mxfp4 import dequantize
    cfg = MoEConfig("mx_slots", T=4, H=256, I=192, E=8, k=2, routed_scale=2.5)
    inp = make_inputs(cfg)
    mw = make_mxfp4_weights(cfg)
    layer, _ = _run(cfg, inp, mw)
    b = layer.last
    perm = b["perm"].cpu().numpy()
    ys = b["y_slots"].float().cpu().numpy()
    w = b["topk_w"].cpu().numpy().reshape(-1)
    idx = b["topk_idx"].cpu().numpy().reshape(-1)
    for p in range(cfg.T * cfg.k):
        q = perm[p]
        t, e = q // cfg.k, idx[q]
        gu = dequantize(mw["gate_up_q"][e].numpy(), mw["gate_up_s"][e].numpy()).astype(np.float32)
        dn = dequantize(mw["down_q"][e].numpy(), mw["down_s"][e].numpy()).astype(np.float32)
        ref = cfg.routed_scale * w[q] * expert(gu, dn, inp["x"][t].double().numpy())
        assert np.linalg.norm(ys[p] - ref) <= BF16_TOL * np.linalg.norm(ref)


def test_mxfp4_matches_bf16_path_on_the_same_values(cuda_ok):
    """The dequantised weights are exact in bf16; the bf16 decode path on them
    and the MXFP4 path agree to the bf16 tolerance."""
    import sparse_mixture_experts_07_b200 as moe
    from oracle.mxfp4 import dequantize
    cfg = MoEConfig("mx_vs_bf16", T=6, H=512, I=256, E=8, k=2)
    inp = make_inputs(cfg)
    mw = make_mxfp4_weights(cfg)
    _, y_mx = _run(cfg, inp, mw)
    d = to_device(inp)
    gu = torch.from_numpy(dequantize(mw["gate_up_q"].numpy(), mw["gate_up_s"].numpy())).to(
        torch.bfloat16).cuda()
    dn = torch.from_numpy(dequantize(mw["down_q"].numpy(), mw["down_s"].numpy())).to(
        torch.bfloat16).cuda()
    layer = moe.MoELayer(moe.Shape.from_config(cfg), d["w_router"], d["router_bias"], gu, dn)
    y_bf = layer(d["x"]).float().cpu()
    torch.cuda.synchronize()
    assert rel_l2(y_mx.float().numpy(), y_bf.numpy()) <= BF16_TOL
