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
    # H and I multiples of 64 but not of 128 (gpt-oss's 2880 is one): the
    # tensor-core kernel on prepared weights (padded rows), a partial last
    # K-group of the activations and, in GEMM 2, a partial last 128-row tile
    MoEConfig("mx_tiled_gptoss_like_T1", T=1, H=320, I=320, E=32, k=4, zipf_s=1.0),
    MoEConfig("mx_tiled_T7", T=7, H=576, I=192, E=16, k=4, routed_scale=2.5),
    MoEConfig("mx_tiled_T33", T=33, H=448, I=320, E=32, k=4, zipf_s=1.0),
    MoEConfig("mx_tiled_T64_splits", T=64, H=2880, I=320, E=8, k=2),
]
# (H, I multiples of 128) run on both weight forms: raw and prepared agree bit for bit
RAW_AND_TILED = [c for c in SMALL if c.H % 128 == 0 and c.I % 128 == 0]


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


@pytest.mark.parametrize("cfg", RAW_AND_TILED, ids=lambda c: c.name)
def test_mxfp4_raw_and_prepared_agree(cuda_ok, cfg):
    """moe_forward_mxfp4 (raw [rows, K/32] scales, per-row copies) and
    moe_forward_mxfp4_prepared (the same scales re-laid out once) run the same
    arithmetic: outputs equal bit for bit; the raw path matches the oracle."""
    import sparse_mixture_experts_07_b200 as moe
    inp = make_inputs(cfg)
    mw = make_mxfp4_weights(cfg)
    layer, y_prep = _run(cfg, inp, mw)
    assert layer.mx_prepared is not None
    b = layer.last
    y_raw = moe.forward_mxfp4(layer.shape, to_device(inp)["x"], b["offsets"], b["perm"],
                              b["topk_w"], layer.mxfp4, layer.workspace, layer.err_flag)
    y_raw = moe.combine(layer.shape, y_raw, b["inv"]).cpu()
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert torch.equal(y_raw, y_prep)
    _check(cfg, inp, mw, layer, y_raw)


def _a256(v):
    return (v + 255) // 256 * 256


def test_mxfp4_prepared_layout(cuda_ok):
    """The prepared array holds, for every (expert, tile, K-group, word, byte),
    the raw scale of the row and block its layout names (127 past the rows
    and blocks), then the codes of both weights with rows padded by zero
    bytes to whole 128-weight groups (H = 320 and I = 192 both need it)."""
    import sparse_mixture_experts_07_b200 as moe
    cfg = MoEConfig("mx_prepare_layout", T=1, H=320, I=192, E=3, k=1)
    mw = make_mxfp4_weights(cfg)
    shape = moe.Shape.from_config(cfg)
    prepared = moe.mxfp4_prepare(shape, {key: v.cuda() for key, v in mw.items()})
    torch.cuda.synchronize()
    got = prepared.cpu().numpy()
    E, H, I = cfg.E, cfg.H, cfg.I
    parts = []
    for gemm in ("gu", "dn"):
        K = H if gemm == "gu" else I
        raw = (mw["gate_up_s"] if gemm == "gu" else mw["down_s"]).numpy()
        mtiles = I // 64 if gemm == "gu" else -(-H // 128)
        atoms = []
        for e in range(E):
            for mt in range(mtiles):
                for kg in range(-(-K // 128)):
                    atom = np.full(512, 127, dtype=np.uint8)
                    for w in range(128):
                        m = (w >> 2) + 32 * (w & 3)
                        if gemm == "gu":
                            row = mt * 64 + m if m < 64 else I + mt * 64 + (m - 64)
                        else:
                            row = mt * 128 + m
                            if row >= H:
                                continue
                        for kb in range(4):
                            blk = 4 * kg + kb
                            if blk < K // 32:
                                atom[4 * w + kb] = raw[e, row, blk]
                    atoms.append(atom)
        parts.append(np.concatenate(atoms))
    for q, K in ((mw["gate_up_q"].numpy(), H), (mw["down_q"].numpy(), I)):
        Kp = -(-K // 128) * 128
        padded = np.zeros(q.shape[:-1] + (Kp // 2,), dtype=np.uint8)
        padded[..., :K // 2] = q
        parts.append(padded.reshape(-1))
    off = 0
    for part in parts:
        assert np.array_equal(got[off:off + part.size], part)
        off = _a256(off + part.size)
    assert off == got.size


@pytest.mark.parametrize("name", ["gptoss_decode1", "gptoss_decode8"])
def test_mxfp4_decode_gptoss_full_size(cuda_ok, name):
    """gpt-oss-shaped layer (H = I = 2880, 32 experts, k = 4): the prepared
    tensor-core path at full size against the oracle."""
    cfg = CONFIGS[name]
    inp = make_inputs(cfg)
    mw = make_mxfp4_weights(cfg)
    layer, y = _run(cfg, inp, mw)
    assert layer.mx_prepared is not None
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
