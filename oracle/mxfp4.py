"""MXFP4 expert weights in the oracle.

TEST INFRASTRUCTURE, like the rest of this package: only tests/,
__graft_entry__.smoke() and bench.py's CPU legs may import it.

"Mixture of Experts in Transformers", section "from dense to sparse": the
gpt-oss experts are stored natively in mxfp4, and a kernel for that format
makes decode faster still.  The pages name the format without defining it.
This module takes the definition of the Open Compute Project Microscaling
(MX) Formats specification v1.0:
  - elements come in blocks of 32 consecutive values along the contraction
    dimension, and each block shares one scale;
  - an element is FP4 E2M1: 1 sign bit, 2 exponent bits with bias 1, and 1
    mantissa bit.  Exponent field 0 is subnormal, (-1)^s * 2^0 * (m / 2);
    otherwise the value is (-1)^s * 2^(e - 1) * (1 + m / 2);
  - a scale is E8M0: an unsigned 8-bit biased exponent, 2^(s - 127); the
    code 255 is NaN.
The element value is the E2M1 value times its block's scale.

Storage (the layout the C ABI takes): a weight matrix of R rows and K columns
(K a multiple of 32) is `q` [R, K/2] uint8, element 2j of a row in the low
nibble of byte j and element 2j+1 in the high nibble, and `s` [R, K/32] uint8.

Everything here is plain numpy in float64; the expert arithmetic is the C
oracle's (`oracle.expert`), fed the dequantised weights.
"""
from __future__ import annotations

import numpy as np

from . import expert, router, topk_softmax

BLOCK = 32


def e2m1(code: int) -> float:
    """Value of a 4-bit E2M1 code (sign, 2-bit exponent with bias 1, 1-bit mantissa)."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = 2.0 ** 0 * (m / 2.0) if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return -mag if s else mag


def e8m0(code: int) -> float:
    """Value of an 8-bit E8M0 scale: 2^(code - 127), NaN for 255."""
    return float("nan") if code == 255 else 2.0 ** (int(code) - 127)


def dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Weights [..., K] in float64 from packed codes q [..., K/2] and scales s [..., K/32]."""
    q = np.asarray(q, dtype=np.uint8)
    s = np.asarray(s, dtype=np.uint8)
    K = q.shape[-1] * 2
    assert s.shape[-1] * BLOCK == K and q.shape[:-1] == s.shape[:-1]
    table = np.array([e2m1(c) for c in range(16)], dtype=np.float64)
    scale = np.array([e8m0(c) for c in range(256)], dtype=np.float64)
    codes = np.empty(q.shape[:-1] + (K,), dtype=np.uint8)
    codes[..., 0::2] = q & 0x0F            # element 2j: low nibble of byte j
    codes[..., 1::2] = q >> 4              # element 2j+1: high nibble
    w = table[codes]
    return w * np.repeat(scale[s], BLOCK, axis=-1)


def moe_block_mxfp4(x, w_router, router_bias, gate_up_q, gate_up_s, down_q, down_s, k: int,
                    routed_scale: float = 1.0, tokens=None):
    """The routed block with MXFP4 expert weights, for the listed tokens (all if None).

    Routing as in the bf16 block (router logits, top-k, softmax over the k);
    each selected expert runs on its dequantised weights; y_t = routed_scale *
    sum_j w_j * FFN_e(x_t).  Returns (y [n, H] float64, idx [n, k], w [n, k])."""
    lg = router(x, w_router, router_bias, tokens=tokens)
    idx, w = topk_softmax(lg, k)
    toks = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    xs = x.float().numpy() if hasattr(x, "float") else np.asarray(x, dtype=np.float64)
    gq, gs = np.asarray(gate_up_q), np.asarray(gate_up_s)
    dq, ds = np.asarray(down_q), np.asarray(down_s)
    y = np.zeros((len(toks), dq.shape[1]), dtype=np.float64)
    # one expert's weights in memory at a time; each token still sums its k
    # expert outputs in the order j = 0..k-1
    outs = {}
    for e in sorted(set(int(v) for v in idx.reshape(-1))):
        # the values are exact in float32 (2-bit significands times 2^(s-127))
        gu_e = dequantize(gq[e], gs[e]).astype(np.float32)
        dn_e = dequantize(dq[e], ds[e]).astype(np.float32)
        for n, t in enumerate(toks):
            for j in range(k):
                if int(idx[n, j]) == e:
                    outs[(n, j)] = expert(gu_e, dn_e, xs[t].astype(np.float64))
    for n in range(len(toks)):
        for j in range(k):
            y[n] += w[n, j] * outs[(n, j)]
    return routed_scale * y, idx, w
