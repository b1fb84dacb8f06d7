"""Pins for the CPU oracle: closed forms, brute force and invariants.

Each test ties one step of the oracle to something other than the oracle's own
code: a value derivable by hand, an exhaustive search, a textbook special case,
or an invariant the method must satisfy (the dropless sparse dispatch equals
the brute-force dense computation; k = E gives the full softmax-weighted sum;
counts sum to T*k; the combine weights of a token sum to 1).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_07_b200.inputs import CONFIGS, MoEConfig, make_inputs

LN3 = math.log(3.0)


def _rand_inputs(T, H, I, E, S=0, Is=0, seed=0, bias=False, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    inp = {
        "x": torch.randn(T, H, generator=g).to(dtype),
        "w_router": torch.randn(E, H, generator=g) * 0.3,
        "router_bias": (torch.randn(E, generator=g) * 0.1) if bias else None,
        "gate_up": (torch.randn(E, 2 * I, H, generator=g) * 0.2).to(dtype),
        "down": (torch.randn(E, H, I, generator=g) * 0.2).to(dtype),
        "sh_gate_up": (torch.randn(S, 2 * Is, H, generator=g) * 0.2).to(dtype) if S else None,
        "sh_down": (torch.randn(S, H, Is, generator=g) * 0.2).to(dtype) if S else None,
    }
    return inp


# ---------------------------------------------------------------- router
def test_router_unit_vectors_give_weight_columns():
    # x = c * e_h  =>  logits[e] = c * Wr[e, h] + b[e]; a transposed Wr fails this.
    H, E = 5, 3
    wr = torch.arange(E * H, dtype=torch.float32).reshape(E, H) / 8.0
    b = torch.tensor([0.5, -1.0, 2.0])
    x = torch.eye(H) * 2.0
    lg = oracle.router(x, wr, b)
    for h in range(H):
        for e in range(E):
            assert lg[h, e] == 2.0 * float(wr[e, h]) + float(b[e])


def test_router_subset_of_tokens():
    inp = _rand_inputs(9, 6, 4, 5)
    full = oracle.router(inp["x"], inp["w_router"])
    part = oracle.router(inp["x"], inp["w_router"], tokens=[7, 2])
    assert np.array_equal(part, full[[7, 2]])


# ---------------------------------------------------------------- top-k + softmax
@pytest.mark.parametrize("k", [1, 2, 3, 6, 8])
def test_topk_is_the_max_sum_subset_in_descending_order(k):
    rng = np.random.default_rng(k)
    E = 8
    logits = rng.normal(size=(40, E))
    idx, w = oracle.topk_softmax(logits, k)
    for r in range(logits.shape[0]):
        best = max(itertools.combinations(range(E), k), key=lambda c: logits[r, list(c)].sum())
        assert sorted(idx[r]) == sorted(best)
        vals = logits[r, idx[r]]
        assert np.all(np.diff(vals) < 0)
        # softmax characterised by: positive, sums to 1, ratios exp(l_i - l_j)
        assert abs(w[r].sum() - 1.0) < 1e-12
        for i in range(k):
            for j in range(k):
                assert math.isclose(w[r, i] / w[r, j], math.exp(vals[i] - vals[j]),
                                    rel_tol=1e-12)


def test_top2_weights_are_sigmoid_of_gap():
    logits = np.array([[0.3, 2.0, -1.0, 1.25]])
    idx, w = oracle.topk_softmax(logits, 2)
    assert list(idx[0]) == [1, 3]
    assert math.isclose(w[0, 0], 1.0 / (1.0 + math.exp(-(2.0 - 1.25))), rel_tol=1e-14)
    assert math.isclose(w[0, 1], 1.0 / (1.0 + math.exp(2.0 - 1.25)), rel_tol=1e-14)


def test_topk_ties_go_to_lower_index():
    logits = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]])
    idx, w = oracle.topk_softmax(logits, 3)
    assert list(idx[0]) == [1, 2, 4]
    assert np.allclose(w[0], 1.0 / 3.0, rtol=0, atol=1e-15)


def test_k_equals_E_gives_full_softmax():
    rng = np.random.default_rng(3)
    logits = rng.normal(size=(10, 6)) * 3
    idx, w = oracle.topk_softmax(logits, 6)
    for r in range(10):
        full = np.zeros(6)
        full[idx[r]] = w[r]
        ref = np.exp(logits[r] - logits[r].max())
        assert np.allclose(full, ref / ref.sum(), rtol=1e-13, atol=0)


# ---------------------------------------------------------------- permutation
def test_permute_matches_stable_sort_and_invariants():
    rng = np.random.default_rng(1)
    T, k, E = 37, 3, 7
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[:, :] = np.where(idx == 6, 5, idx)          # leave expert 6 empty
    idx = np.stack([np.array(sorted(set(r)) + [c for c in range(E) if c not in r][:k - len(set(r))])
                    for r in idx]).astype(np.int32)
    counts, offsets, perm, inv = oracle.permute(idx, E)
    slots = idx.reshape(-1)
    ref = sorted(range(T * k), key=lambda q: (slots[q], q))
    assert list(perm) == ref
    assert counts.sum() == T * k
    assert list(counts) == [int((slots == e).sum()) for e in range(E)]
    assert offsets[0] == 0 and list(np.diff(offsets)) == list(counts)
    assert np.array_equal(inv[perm], np.arange(T * k))


def test_permute_rejects_out_of_range_index():
    with pytest.raises(RuntimeError):
        oracle.permute(np.array([[0, 4]], dtype=np.int32), 4)


# ---------------------------------------------------------------- expert FFN
def test_expert_scalar_closed_form():
    # H = I = 1: out = d * SiLU(g x) * (u x); SiLU(ln 3) = (3/4) ln 3 exactly.
    gu = torch.tensor([[1.0], [2.0]])
    dn = torch.tensor([[0.5]])
    out = oracle.expert(gu, dn, np.array([LN3]))
    assert math.isclose(out[0], 0.5 * 0.75 * LN3 * 2.0 * LN3, rel_tol=1e-14)
    # SiLU(0) = 0 and SiLU(-ln 3) = -(1/4) ln 3
    assert oracle.expert(gu, dn, np.array([0.0]))[0] == 0.0
    assert math.isclose(oracle.expert(gu, dn, np.array([-LN3]))[0],
                        0.5 * (-0.25 * LN3) * 2.0 * (-LN3), rel_tol=1e-14)


def test_expert_gate_up_order_and_down_orientation():
    # x = [ln3, 0]; gate rows g0 = +1, g1 = -1 (times x0); up rows 2, 4.
    # a = [SiLU(ln3)*2 ln3, SiLU(-ln3)*4 ln3] = [1.5 ln3^2, -ln3^2]
    # down = [[1,2],[3,7]] -> out = [1.5-2, 4.5-7] * ln3^2 = [-0.5, -2.5] ln3^2
    gu = torch.tensor([[1.0, 0.0], [-1.0, 0.0], [2.0, 0.0], [4.0, 0.0]])
    dn = torch.tensor([[1.0, 2.0], [3.0, 7.0]])
    out = oracle.expert(gu, dn, np.array([LN3, 0.0]))
    L = LN3 * LN3
    assert math.isclose(out[0], -0.5 * L, rel_tol=1e-13)
    assert math.isclose(out[1], -2.5 * L, rel_tol=1e-13)


def test_single_expert_is_textbook_swiglu():
    # E = 1, k = 1: the block is down(SiLU(gate x) * up x), routing weight 1.
    T, H, I = 6, 10, 7
    inp = _rand_inputs(T, H, I, 1, seed=4)
    y, idx, w = oracle.moe_block(inp, k=1)
    assert np.all(idx == 0) and np.all(w == 1.0)
    x = inp["x"].double().numpy()
    gu = inp["gate_up"][0].double().numpy()
    dn = inp["down"][0].double().numpy()
    g, u = x @ gu[:I].T, x @ gu[I:].T
    ref = (g * (1.0 / (1.0 + np.exp(-g))) * u) @ dn.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- the block
def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("S", [0, 2])
def test_sparse_equals_dense_bruteforce(dtype, S):
    inp = _rand_inputs(24, 16, 12, 6, S=S, Is=8, seed=5, bias=True, dtype=dtype)
    for k in (1, 2, 4):
        y, _, _ = oracle.moe_block(inp, k=k, routed_scale=2.5 if S else 1.0)
        yd = oracle.moe_dense(inp, k=k, routed_scale=2.5 if S else 1.0)
        assert _rel_l2(y, yd) < 1e-13


def test_tiny_config_sparse_equals_dense():
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=0)
    y, idx, w = oracle.moe_block(inp, k=cfg.k)
    yd = oracle.moe_dense(inp, k=cfg.k)
    assert _rel_l2(y, yd) < 1e-13
    counts, offsets, perm, inv = oracle.permute(idx, cfg.E)
    assert counts.sum() == cfg.T * cfg.k
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)


def test_k_equals_E_block_is_full_weighted_sum():
    T, H, I, E = 5, 8, 6, 4
    inp = _rand_inputs(T, H, I, E, seed=6, bias=True)
    y, _, _ = oracle.moe_block(inp, k=E)
    logits = oracle.router(inp["x"], inp["w_router"], inp["router_bias"])
    for t in range(T):
        p = np.exp(logits[t] - logits[t].max())
        p /= p.sum()
        xv = inp["x"][t].double().numpy()
        ref = sum(p[e] * oracle.expert(inp["gate_up"][e], inp["down"][e], xv) for e in range(E))
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-14)


def test_shared_experts_split_equals_merged():
    # Two shared experts of width Is == one shared expert of width 2 Is whose
    # gate rows, up rows and down columns are the concatenations.
    T, H, I, E, Is = 7, 12, 5, 4, 6
    inp = _rand_inputs(T, H, I, E, S=2, Is=Is, seed=7)
    gu, dn = inp["sh_gate_up"], inp["sh_down"]
    merged = dict(inp)
    merged["sh_gate_up"] = torch.cat([gu[0, :Is], gu[1, :Is], gu[0, Is:], gu[1, Is:]])[None]
    merged["sh_down"] = torch.cat([dn[0], dn[1]], dim=1)[None]
    y1, _, _ = oracle.moe_block(inp, k=2, routed_scale=2.5)
    y2, _, _ = oracle.moe_block(merged, k=2, routed_scale=2.5)
    assert np.allclose(y1, y2, rtol=1e-12, atol=1e-14)


def test_zero_routed_scale_leaves_only_shared():
    T, H, I, E, Is = 4, 8, 5, 3, 6
    inp = _rand_inputs(T, H, I, E, S=2, Is=Is, seed=8)
    y, _, _ = oracle.moe_block(inp, k=2, routed_scale=0.0)
    for t in range(T):
        xv = inp["x"][t].double().numpy()
        ref = sum(oracle.expert(inp["sh_gate_up"][s], inp["sh_down"][s], xv) for s in range(2))
        assert np.allclose(y[t], ref, rtol=1e-13, atol=1e-15)


def test_routed_scale_is_linear_in_routed_part():
    inp = _rand_inputs(6, 8, 5, 4, S=1, Is=4, seed=9)
    y0, _, _ = oracle.moe_block(inp, k=2, routed_scale=0.0)
    y1, _, _ = oracle.moe_block(inp, k=2, routed_scale=1.0)
    y25, _, _ = oracle.moe_block(inp, k=2, routed_scale=2.5)
    assert np.allclose(y25 - y0, 2.5 * (y1 - y0), rtol=1e-12, atol=1e-14)


def test_hand_worked_block():
    # x = [1, 0]; Wr rows [2,0], [1,0], [0,0]  ->  logits [2, 1, 0], top-2 = (0, 1),
    # weights (sigmoid(1), sigmoid(-1)).  Expert e: gate row [g_e, 0], up row [u_e, 0],
    # down column [d_e0, d_e1].  Expert 0: g = ln3 -> SiLU = 0.75 ln3, u = 2.
    # Expert 1: g = -ln3 -> SiLU = -0.25 ln3, u = 4.  Expert 2 is never used.
    x = torch.tensor([[1.0, 0.0]])
    wr = torch.tensor([[2.0, 0.0], [1.0, 0.0], [0.0, 0.0]])
    gu = torch.tensor([[[LN3, 0.0], [2.0, 0.0]], [[-LN3, 0.0], [4.0, 0.0]],
                       [[9.0, 9.0], [9.0, 9.0]]])
    dn = torch.tensor([[[1.0], [3.0]], [[2.0], [7.0]], [[9.0], [9.0]]])
    inp = {"x": x, "w_router": wr, "router_bias": None, "gate_up": gu, "down": dn}
    y, idx, w = oracle.moe_block(inp, k=2, routed_scale=2.5)
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    a0, a1 = 0.75 * LN3 * 2.0, -0.25 * LN3 * 4.0
    ref = 2.5 * (s1 * a0 * np.array([1.0, 3.0]) + (1.0 - s1) * a1 * np.array([2.0, 7.0]))
    assert list(idx[0]) == [0, 1]
    assert np.allclose(w[0], [s1, 1.0 - s1], rtol=1e-15)
    # the weights are float32-rounded ln3 values: allow their relative rounding
    assert np.allclose(y[0], ref, rtol=1e-6, atol=0)


def test_token_permutation_permutes_rows():
    inp = _rand_inputs(11, 8, 6, 5, S=1, Is=4, seed=10, bias=True)
    y, idx, w = oracle.moe_block(inp, k=2)
    pi = np.random.default_rng(0).permutation(11)
    inp2 = dict(inp)
    inp2["x"] = inp["x"][torch.from_numpy(pi)]
    y2, idx2, w2 = oracle.moe_block(inp2, k=2)
    assert np.array_equal(idx2, idx[pi])
    assert np.allclose(y2, y[pi], rtol=1e-14, atol=0)


def test_constant_logit_shift_leaves_routing_unchanged():
    inp = _rand_inputs(13, 8, 6, 5, seed=11)
    y, idx, w = oracle.moe_block(inp, k=3)
    inp2 = dict(inp)
    inp2["router_bias"] = torch.full((5,), 0.75)
    y2, idx2, w2 = oracle.moe_block(inp2, k=3)
    assert np.array_equal(idx, idx2)
    assert np.allclose(w, w2, rtol=1e-12)
    assert np.allclose(y, y2, rtol=1e-11)


def test_bf16_storage_is_widened_exactly():
    inp = _rand_inputs(9, 8, 6, 4, S=1, Is=4, seed=12, dtype=torch.bfloat16)
    as_f32 = {kk: (v.float() if isinstance(v, torch.Tensor) else v) for kk, v in inp.items()}
    y1, i1, _ = oracle.moe_block(inp, k=2)
    y2, i2, _ = oracle.moe_block(as_f32, k=2)
    assert np.array_equal(i1, i2) and np.array_equal(y1, y2)


# ---------------------------------------------------------------- page-printed shapes
def _golden_shapes():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "page_model_shapes.txt")
    vals = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            key, val = line.split()[:2]
            vals[key] = float(val)
    return vals


def test_configs_follow_page_shapes():
    g = _golden_shapes()
    ph = CONFIGS["phimoe_prefill"]
    assert (ph.H, ph.I, ph.E, ph.k) == (g["phimoe.hidden_size"], g["phimoe.intermediate_size"],
                                        g["phimoe.num_local_experts"],
                                        g["phimoe.num_experts_per_tok"])
    for n in ("phimoe_decode1", "phimoe_decode8", "phimoe_decode64"):
        c = CONFIGS[n]
        assert (c.H, c.I, c.E, c.k) == (ph.H, ph.I, ph.E, ph.k)
    go = CONFIGS["gptoss"]
    assert (go.E, go.k) == (g["gptoss.num_experts"], g["gptoss.active_experts"])
    ds = CONFIGS["dsv3"]
    assert (ds.E, ds.n_shared, ds.k, ds.routed_scale, ds.H) == (
        g["instella.routed_experts"], g["instella.shared_experts"],
        g["instella.num_experts_per_tok"], g["instella.routed_scaling_factor"],
        g["instella.hidden_size"])
    assert CONFIGS["mixtral"].k == g["mixtral.num_experts_per_tok"]
    from sparse_mixture_experts_07_b200.inputs import INIT_STD
    assert INIT_STD == g["phimoe.initializer_range"]


# ------------------------------------------------- expert-parallel partials
@pytest.mark.parametrize("bounds", [(0, 2, 4, 6), (0, 1, 6), (0, 3, 3, 6), (0, 6)])
def test_expert_partials_over_a_partition_sum_to_the_block(bounds):
    """The ranks' partials (each its range of experts, shared experts on the
    first rank only) sum to the whole block; a rank without experts and
    without the shared experts contributes zero."""
    inp = _rand_inputs(10, 12, 8, 6, S=2, Is=5, seed=11, bias=True)
    y, _, _ = oracle.moe_block(inp, k=3, routed_scale=2.5)
    parts = [oracle.moe_block_experts(inp, k=3, routed_scale=2.5, e_begin=a, e_end=b,
                                      with_shared=(r == 0))
             for r, (a, b) in enumerate(zip(bounds[:-1], bounds[1:]))]
    assert _rel_l2(sum(parts), y) < 1e-13
    for (a, b), part in zip(zip(bounds[:-1], bounds[1:]), parts):
        if a == b and part is not parts[0]:
            assert not part.any()


def test_expert_partial_of_one_expert_is_its_weighted_output():
    inp = _rand_inputs(6, 8, 5, 4, seed=12, bias=True)
    lg = oracle.router(inp["x"], inp["w_router"], inp["router_bias"])
    idx, w = oracle.topk_softmax(lg, 2)
    part = oracle.moe_block_experts(inp, k=2, routed_scale=1.0, e_begin=1, e_end=2)
    for t in range(6):
        ref = np.zeros(8)
        for j in range(2):
            if idx[t, j] == 1:
                ref = w[t, j] * oracle.expert(inp["gate_up"][1], inp["down"][1],
                                              inp["x"][t].double().numpy())
        assert np.allclose(part[t], ref, rtol=1e-13, atol=1e-15)


# ---------------------------------------------- DeepSeek-V3 (noaux_tc) routing
def _sigmoid(v):
    return 1.0 / (1.0 + math.exp(-v))


def test_noaux_without_groups_or_bias_is_topk_of_the_logits():
    """One group and no bias: sigmoid is increasing, so the selection is the
    plain top-k of the logits, and the weights are the selected sigmoids
    normalised."""
    rng = np.random.default_rng(21)
    lg = rng.normal(size=(40, 16))
    idx, w = oracle.route_noaux_tc(lg, None, 4, 1, 1)
    idx_ref, _ = oracle.topk_softmax(lg, 4)
    assert np.array_equal(idx, idx_ref)
    for t in range(40):
        s = np.array([_sigmoid(lg[t, e]) for e in idx[t]])
        assert np.allclose(w[t], s / s.sum(), rtol=1e-14, atol=0)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)


def test_noaux_bias_moves_the_selection_but_not_the_weights():
    lg = np.array([[2.0, 1.0, 0.0, -1.0]])
    bias = np.array([0.0, 0.0, 0.0, 5.0], dtype=np.float32)
    idx, w = oracle.route_noaux_tc(lg, bias, 2, 1, 1)
    assert idx.tolist() == [[3, 0]]            # 5 + sigmoid(-1) first, then sigmoid(2)
    s3, s0 = _sigmoid(-1.0), _sigmoid(2.0)
    assert np.allclose(w[0], [s3 / (s3 + s0), s0 / (s3 + s0)], rtol=1e-14, atol=0)


def test_noaux_hand_worked_group_limited_selection():
    """E=8 in 4 groups of 2, keep 2 groups, k=3.  Affinities (sigmoid of the
    logits) 0.953 0.047 | 0.881 0.870 | 0.924 0.018 | 0.500 0.525; group scores
    (sums) 1.000, 1.751, 0.942, 1.025, so groups 1 and 3 are kept and the two
    largest affinities overall (experts 0 and 4) are excluded."""
    lg = np.array([[3.0, -3.0, 2.0, 1.9, 2.5, -4.0, 0.0, 0.1]])
    idx, w = oracle.route_noaux_tc(lg, None, 3, 4, 2)
    assert idx.tolist() == [[2, 3, 7]]
    s = np.array([_sigmoid(2.0), _sigmoid(1.9), _sigmoid(0.1)])
    assert np.allclose(w[0], s / s.sum(), rtol=1e-14, atol=0)
    # keeping every group removes the restriction: the plain top-3
    idx_all, _ = oracle.route_noaux_tc(lg, None, 3, 4, 4)
    assert idx_all.tolist() == [[0, 4, 2]]


def test_noaux_keeping_all_groups_equals_one_group():
    rng = np.random.default_rng(22)
    lg = rng.normal(size=(30, 24))
    bias = rng.normal(scale=0.3, size=24).astype(np.float32)
    a = oracle.route_noaux_tc(lg, bias, 5, 1, 1)
    b = oracle.route_noaux_tc(lg, bias, 5, 6, 6)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_noaux_selected_experts_lie_in_the_best_groups():
    """With 8 groups of 8 and 4 kept, every selected expert's group is among
    the 4 groups with the largest two-expert sums; permuting whole groups
    permutes the selection with them."""
    rng = np.random.default_rng(23)
    E, G, kg, k = 64, 8, 4, 6
    lg = rng.normal(size=(50, E))
    bias = rng.normal(scale=0.2, size=E).astype(np.float32)
    idx, _ = oracle.route_noaux_tc(lg, bias, k, G, kg)
    c = 1.0 / (1.0 + np.exp(-lg)) + bias.astype(np.float64)
    gs = np.sort(c.reshape(50, G, E // G), axis=2)[:, :, -2:].sum(axis=2)
    kept = np.argsort(-gs, axis=1)[:, :kg]
    for t in range(50):
        assert set((idx[t] // (E // G)).tolist()) <= set(kept[t].tolist())
    order = rng.permutation(G)
    cols = np.concatenate([np.arange(g * 8, g * 8 + 8) for g in order])
    idx2, _ = oracle.route_noaux_tc(lg[:, cols], bias[cols], k, G, kg)
    assert np.array_equal(cols[idx2], idx)


def test_routed_block_with_softmax_routing_is_the_block():
    inp = _rand_inputs(9, 12, 8, 6, S=1, Is=5, seed=24, bias=True)
    y, idx, w = oracle.moe_block(inp, k=2, routed_scale=2.5)
    y2 = oracle.moe_block_routed(inp, idx, w, routed_scale=2.5)
    assert _rel_l2(y2, y) < 1e-14
    toks = [8, 0, 3]
    y3 = oracle.moe_block_routed(inp, idx[toks], w[toks], routed_scale=2.5, tokens=toks)
    assert _rel_l2(y3, y[toks]) < 1e-14


# ------------------------------------------------------------ backward pass
def _loss(inp, k, dy, scale):
    y, _, _ = oracle.moe_block(inp, k=k, routed_scale=scale)
    return float((y * dy).sum())


def _fd_check(inp, name, k, dy, scale, grad, n_pick, rng, delta=2.0 ** -12):
    """Central differences of L = <dy, y> against the analytic gradient, on
    n_pick random entries of the float32 tensor inp[name]; each perturbation
    is a power of two, exact in float32, so the difference quotient is
    float64-accurate up to O(delta^2)."""
    t = inp[name]
    flat = t.view(-1)
    for i in rng.choice(flat.numel(), size=min(n_pick, flat.numel()), replace=False):
        old = float(flat[i])
        flat[i] = old + delta
        lp = _loss(inp, k, dy, scale)
        flat[i] = old - delta
        lm = _loss(inp, k, dy, scale)
        flat[i] = old
        fd = (lp - lm) / (2 * delta)
        g = float(grad.reshape(-1)[i])
        assert abs(fd - g) <= 1e-6 * max(1.0, abs(g)) + 1e-9, (name, int(i), fd, g)


@pytest.mark.parametrize("S", [0, 2])
def test_backward_matches_finite_differences(S):
    """Every gradient the oracle's backward returns (x, both expert weights,
    router weight and bias, shared experts) agrees with central finite
    differences of its own forward: an independent check of the chain rule."""
    inp = _rand_inputs(6, 8, 5, 4, S=S, Is=3, seed=31, bias=True)
    scale = 2.5 if S else 1.0
    rng = np.random.default_rng(31)
    dy = rng.normal(size=(6, 8))
    gr = oracle.moe_backward(inp, 2, dy, routed_scale=scale)
    names = ["x", "gate_up", "down", "w_router", "router_bias"]
    if S:
        names += ["sh_gate_up", "sh_down"]
    for name in names:
        _fd_check(inp, name, 2, dy, scale, gr[name], 24, rng)


def test_backward_routing_weight_and_logit_gradients():
    """dw_j = s <dy, f_j> (each expert's output read back from the block with
    a one-hot weight) and dl is the softmax Jacobian over the selected k
    applied to dw: zero off the selection, summing to zero per token."""
    inp = _rand_inputs(5, 8, 6, 5, seed=32, bias=True)
    rng = np.random.default_rng(32)
    dy = rng.normal(size=(5, 8))
    gr = oracle.moe_backward(inp, 3, dy, routed_scale=2.0)
    y, idx, w = oracle.moe_block(inp, k=3, routed_scale=2.0)
    for t in range(5):
        xv = inp["x"][t].double().numpy()
        for j in range(3):
            f = oracle.expert(inp["gate_up"][idx[t, j]], inp["down"][idx[t, j]], xv)
            assert np.isclose(gr["dw"][t, j], 2.0 * float(dy[t] @ f), rtol=1e-12, atol=1e-14)
        off = np.setdiff1d(np.arange(5), idx[t])
        assert np.all(gr["dl"][t, off] == 0.0)
        assert abs(gr["dl"][t].sum()) < 1e-14
    assert np.allclose(gr["router_bias"], gr["dl"].sum(axis=0), rtol=1e-13, atol=1e-15)


def test_aux_loss_closed_forms_and_finite_differences():
    T, E, k = 12, 6, 2
    rng = np.random.default_rng(33)
    # uniform router: p = 1/E, so the loss is coef * k and dl = coef/T (f - k/E)
    lg = np.zeros((T, E))
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    loss, dl = oracle.aux_loss(lg, idx, E, coef=0.01)
    f = np.bincount(idx.reshape(-1), minlength=E) / T
    assert np.isclose(loss, 0.01 * k, rtol=1e-14)
    assert np.allclose(dl, 0.01 / T * (f - k / E)[None, :], rtol=1e-13, atol=1e-17)
    # random logits: central differences (the dispatch counts held fixed)
    lg = rng.normal(size=(T, E))
    loss, dl = oracle.aux_loss(lg, idx, E, coef=0.01)
    for t, e in [(0, 0), (3, 5), (11, 2), (7, 1)]:
        d = 1e-6
        lp, lm = lg.copy(), lg.copy()
        lp[t, e] += d
        lm[t, e] -= d
        fd = (oracle.aux_loss(lp, idx, E, 0.01)[0] - oracle.aux_loss(lm, idx, E, 0.01)[0]) / (2 * d)
        assert abs(fd - dl[t, e]) <= 1e-9
