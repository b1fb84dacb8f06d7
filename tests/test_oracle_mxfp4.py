"""Pins of the oracle's MXFP4 expert weights (oracle/mxfp4.py).

The pages name mxfp4 as gpt-oss's native expert format ("Mixture of Experts in
Transformers", section "from dense to sparse") without defining it; the
definition is the OCP Microscaling (MX) Formats specification v1.0.  Each pin
ties the oracle to that definition or to plain float64 algebra."""
import math

import numpy as np
import torch

import oracle
from oracle import mxfp4
from sparse_mixture_experts_07_b200.inputs import MoEConfig, make_inputs, make_mxfp4_weights

# FP4 E2M1 values by code, as tabulated in the OCP MX specification v1.0
# (element data types): magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign.
E2M1_SPEC = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
             -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_codes_match_the_specification_table():
    for code, v in enumerate(E2M1_SPEC):
        got = mxfp4.e2m1(code)
        assert got == v and math.copysign(1.0, got) == math.copysign(1.0, v)


def test_e8m0_scale_is_a_power_of_two_with_nan_at_255():
    assert mxfp4.e8m0(127) == 1.0
    assert mxfp4.e8m0(128) == 2.0
    assert mxfp4.e8m0(0) == 2.0 ** -127
    assert mxfp4.e8m0(254) == 2.0 ** 127
    assert math.isnan(mxfp4.e8m0(255))


def test_nibble_order_and_block_scale():
    # byte 0x21: element 0 is the low nibble (code 1 = 0.5), element 1 the high
    # nibble (code 2 = 1.0); the block's scale 128 doubles both
    q = np.zeros((1, 16), dtype=np.uint8)
    q[0, 0] = 0x21
    q[0, 15] = 0xF9          # elements 30, 31: codes 9 (-0.5) and 15 (-6)
    w = mxfp4.dequantize(q, np.array([[128]], dtype=np.uint8))
    assert w.shape == (1, 32)
    assert w[0, 0] == 1.0 and w[0, 1] == 2.0
    assert w[0, 30] == -1.0 and w[0, 31] == -12.0
    assert np.all(w[0, 2:30] == 0.0)


def test_each_block_takes_its_own_scale():
    codes = np.array([2] * 64, dtype=np.uint8)              # every element 1.0
    q = (codes[0::2] | (codes[1::2] << 4)).reshape(1, 32)
    w = mxfp4.dequantize(q, np.array([[125, 130]], dtype=np.uint8))
    assert np.all(w[0, :32] == 0.25) and np.all(w[0, 32:] == 8.0)


def test_single_mxfp4_expert_is_textbook_swiglu():
    """E = 1, k = 1: the block is down(SiLU(gate x) * up x) on the dequantised
    weights, written here with numpy float64 matmuls (gate rows first)."""
    cfg = MoEConfig("mx1", T=3, H=64, I=96, E=1, k=1)
    inp = make_inputs(cfg)
    mw = make_mxfp4_weights(cfg, seed=5)
    y, idx, w = mxfp4.moe_block_mxfp4(inp["x"], inp["w_router"], None, mw["gate_up_q"],
                                      mw["gate_up_s"], mw["down_q"], mw["down_s"], k=1)
    gu = mxfp4.dequantize(mw["gate_up_q"][0].numpy(), mw["gate_up_s"][0].numpy())
    dn = mxfp4.dequantize(mw["down_q"][0].numpy(), mw["down_s"][0].numpy())
    x = inp["x"].double().numpy()
    g, u = x @ gu[:cfg.I].T, x @ gu[cfg.I:].T
    ref = (g / (1.0 + np.exp(-g)) * u) @ dn.T
    assert np.all(idx == 0) and np.allclose(w, 1.0)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_mxfp4_block_equals_bf16_block_on_the_same_values():
    """The dequantised values are exact in bf16 (2-bit significands, scales
    2^-8 and 2^-7), so the MXFP4 block equals the bf16 block on those values."""
    cfg = MoEConfig("mx_vs_bf16", T=40, H=128, I=64, E=6, k=2)
    inp = make_inputs(cfg)
    mw = make_mxfp4_weights(cfg, seed=1)
    gu = mxfp4.dequantize(mw["gate_up_q"].numpy(), mw["gate_up_s"].numpy())
    dn = mxfp4.dequantize(mw["down_q"].numpy(), mw["down_s"].numpy())
    gu_bf = torch.from_numpy(gu).to(torch.bfloat16)
    dn_bf = torch.from_numpy(dn).to(torch.bfloat16)
    assert np.array_equal(gu_bf.double().numpy(), gu) and np.array_equal(dn_bf.double().numpy(), dn)
    y_mx, idx_mx, _ = mxfp4.moe_block_mxfp4(inp["x"], inp["w_router"], inp["router_bias"],
                                            mw["gate_up_q"], mw["gate_up_s"], mw["down_q"],
                                            mw["down_s"], k=cfg.k, routed_scale=2.5)
    ref_inp = dict(inp, gate_up=gu_bf, down=dn_bf)
    y_bf, idx_bf, _ = oracle.moe_block(ref_inp, k=cfg.k, routed_scale=2.5)
    assert np.array_equal(idx_mx, idx_bf)
    assert np.allclose(y_mx, y_bf, rtol=1e-12, atol=1e-15)


def test_generated_weights_have_the_initializer_scale():
    cfg = MoEConfig("mx_rms", T=1, H=256, I=128, E=2, k=1)
    mw = make_mxfp4_weights(cfg)
    w = mxfp4.dequantize(mw["gate_up_q"].numpy(), mw["gate_up_s"].numpy())
    assert 0.015 < float(np.sqrt(np.mean(w * w))) < 0.03
