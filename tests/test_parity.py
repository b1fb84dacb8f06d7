"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Routing indices, counts, offsets and the permutation are
compared bit-exactly; outputs by relative L2 error (1e-5 float32, 1e-2 bf16).
"""
import numpy as np
import pytest
import torch

from parity_util import (check_outputs, check_routing, run_gpu, stratified_tokens,
                         to_device)
from sparse_mixture_experts_07_b200.inputs import CONFIGS, MoEConfig, make_inputs

pytestmark = pytest.mark.gpu

# Small shapes the oracle finishes in seconds; each spans several tiles and has
# ragged tails in rows (experts' counts), in N and in K.
SMALL = [
    MoEConfig("f32_small", T=200, H=136, I=200, E=8, k=2, dtype="f32"),
    MoEConfig("f32_shared", T=77, H=64, I=96, E=6, k=3, n_shared=2, I_shared=40,
              routed_scale=2.5, dtype="f32", zipf_s=1.0),
    MoEConfig("bf16_tiles", T=300, H=512, I=384, E=8, k=2),
    MoEConfig("bf16_ragged", T=333, H=712, I=328, E=8, k=2),
    MoEConfig("bf16_many_experts", T=256, H=256, I=136, E=64, k=6, n_shared=2, I_shared=128,
              routed_scale=2.5, zipf_s=1.2),
    MoEConfig("bf16_gptoss_like", T=512, H=360, I=360, E=32, k=4, zipf_s=1.0),
    MoEConfig("bf16_empty_experts", T=5, H=256, I=128, E=16, k=1),
    MoEConfig("bf16_one_token", T=1, H=512, I=256, E=16, k=2),
    MoEConfig("bf16_k_equals_E", T=40, H=128, I=128, E=4, k=4),
    # > 256 tokens: tensor-core router (E <= 64) or CUDA-core tiled router
    MoEConfig("f32_many_tokens", T=600, H=72, I=64, E=8, k=2, dtype="f32"),
    MoEConfig("bf16_E128", T=300, H=128, I=64, E=128, k=4),
    # decode-batch router cluster with the router slice read from memory (E x H/8
    # floats do not fit in shared memory), 256 experts
    MoEConfig("bf16_route_cluster_E256", T=20, H=2048, I=64, E=256, k=8),
    MoEConfig("bf16_router_tc_E40", T=520, H=200, I=64, E=40, k=3, zipf_s=1.0),
    # decode batches (T <= 8) take the weight-streaming path; ragged H, I, Is
    MoEConfig("bf16_decode_shared", T=7, H=712, I=328, E=16, k=3, n_shared=2, I_shared=200,
              routed_scale=2.5),
    MoEConfig("bf16_decode_T8", T=8, H=1024, I=512, E=4, k=4),
    MoEConfig("bf16_just_above_decode", T=9, H=256, I=256, E=8, k=2),
    # >= 256 rows per expert on average: CTA-pair kernel, incl. 64-row-per-CTA
    # half tiles for group tails of <= 128 rows, ragged N and K, shared experts
    MoEConfig("pair_ragged", T=1100, H=712, I=328, E=4, k=2),
    MoEConfig("pair_shared_zipf", T=600, H=256, I=256, E=4, k=2, n_shared=2, I_shared=136,
              routed_scale=2.5, zipf_s=1.0),
    MoEConfig("pair_many_groups", T=1536, H=384, I=200, E=12, k=3, zipf_s=1.2),
]


def _run(cfg, weights_device="cuda"):
    inp = make_inputs(cfg, seed=0, weights_device="cpu")
    res = run_gpu(cfg, to_device(inp))
    return inp, res


def test_tiny_config_full_parity(cuda_ok):
    cfg = CONFIGS["tiny"]
    inp, res = _run(cfg)
    assert res["err"] == 0
    check_routing(cfg, inp, res)
    err = check_outputs(cfg, inp, res)
    assert err < 1e-5


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_configs(cuda_ok, cfg):
    inp, res = _run(cfg)
    assert res["err"] == 0
    check_routing(cfg, inp, res)
    check_outputs(cfg, inp, res)


SHARED = [c for c in SMALL if c.n_shared > 1]


@pytest.mark.parametrize("cfg", SHARED, ids=lambda c: c.name)
def test_shared_experts_merged_and_separate(cuda_ok, cfg):
    """Two shared experts run as one merged expert (the layer's default) and as
    separate groups: both match the oracle, whose shared experts stay
    separate; the routed slot rows are the same bits either way."""
    inp = make_inputs(cfg, seed=0, weights_device="cpu")
    d = to_device(inp)
    merged = run_gpu(cfg, d)
    separate = run_gpu(cfg, d, merge_shared=False)
    tk = cfg.T * cfg.k
    assert merged["y_slots"].shape[0] == cfg.T * (cfg.k + 1)
    assert separate["y_slots"].shape[0] == cfg.T * (cfg.k + cfg.n_shared)
    assert torch.equal(merged["y_slots"][:tk], separate["y_slots"][:tk])
    for res in (merged, separate):
        assert res["err"] == 0
        check_routing(cfg, inp, res)
        check_outputs(cfg, inp, res)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_shared_merge_layout(cuda_ok, dtype):
    """moe_shared_merge stacks the experts' gate rows, then their up rows, and
    concatenates their down matrices along the columns."""
    import sparse_mixture_experts_07_b200 as moe
    S, Is, H = 3, 40, 24
    shape = moe.Shape(T=4, H=H, I=16, E=4, k=2, n_shared=S, I_shared=Is,
                      dtype=moe.MOE_BF16 if dtype == "bf16" else moe.MOE_F32)
    g = torch.Generator().manual_seed(1)
    gu = torch.randn(S, 2 * Is, H, generator=g).to(shape.torch_dtype)
    dn = torch.randn(S, H, Is, generator=g).to(shape.torch_dtype)
    m_shape, m_gu, m_dn = moe.shared_merge(shape, gu.cuda(), dn.cuda())
    torch.cuda.synchronize()
    assert (m_shape.n_shared, m_shape.I_shared) == (1, S * Is)
    want_gu = torch.cat([gu[:, :Is].reshape(S * Is, H), gu[:, Is:].reshape(S * Is, H)])
    want_dn = torch.cat([dn[e] for e in range(S)], dim=1)
    assert torch.equal(m_gu.cpu()[0], want_gu)
    assert torch.equal(m_dn.cpu()[0], want_dn)


def test_routed_slot_rows_hold_weighted_expert_outputs(cuda_ok):
    # y_slots row p = routed_scale * w * FFN_e(x_t) for slot perm[p]
    import oracle
    cfg = MoEConfig("slots", T=64, H=256, I=256, E=8, k=2, n_shared=1, I_shared=128,
                    routed_scale=2.5)
    inp, res = _run(cfg)
    perm = res["perm"].numpy()
    ys = res["y_slots"].float().numpy()
    w = res["topk_w"].numpy().reshape(-1)
    idx = res["topk_idx"].numpy().reshape(-1)
    for p in (0, 5, 63, 100, cfg.T * cfg.k - 1):
        q = perm[p]
        t, e = q // cfg.k, idx[q]
        ref = cfg.routed_scale * w[q] * oracle.expert(inp["gate_up"][e], inp["down"][e],
                                                      inp["x"][t].double().numpy())
        assert np.linalg.norm(ys[p] - ref) <= 1e-2 * np.linalg.norm(ref)
    for t in (0, 31, 63):
        ref = oracle.expert(inp["sh_gate_up"][0], inp["sh_down"][0], inp["x"][t].double().numpy())
        row = ys[cfg.T * cfg.k + t]
        assert np.linalg.norm(row - ref) <= 1e-2 * np.linalg.norm(ref)


def test_repeat_runs_are_bit_identical(cuda_ok):
    cfg = MoEConfig("det", T=1000, H=256, I=256, E=16, k=4, zipf_s=1.0)
    inp = to_device(make_inputs(cfg))
    a = run_gpu(cfg, inp)
    b = run_gpu(cfg, inp)
    for key in ("topk_idx", "perm", "y"):
        assert torch.equal(a[key], b[key])


def test_bad_expert_index_sets_error_flag(cuda_ok):
    import sparse_mixture_experts_07_b200 as moe
    shape = moe.Shape(T=8, H=128, I=128, E=4, k=2)
    idx = torch.tensor([[0, 1]] * 7 + [[2, 9]], dtype=torch.int32, device="cuda")
    ws = moe.alloc_workspace(shape)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    counts, offsets, perm, inv = moe.permute(shape, idx, ws, err)
    torch.cuda.synchronize()
    assert err.item() == 1 << 5
    assert int(counts.sum()) == 15


FULL = ["mixtral", "phimoe_prefill", "gptoss", "dsv3", "phimoe_decode1", "phimoe_decode8",
        "phimoe_decode64"]

# Tokens whose outputs are checked against the oracle at full size: every
# routed expert's first row, the first and last row of its last 128-row tile
# and two more of its rows, then random tokens up to this many (about 15-25 s
# of oracle time each on 16 host cores).
FULL_SAMPLE = {"mixtral": 768, "phimoe_prefill": 1024, "gptoss": 2048, "dsv3": 2048}


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(cuda_ok, name):
    """Full-size configurations: routing for every token, the plan bit-exact
    against the oracle's, and the outputs of a stratified sample of tokens
    (all tokens of the decode batches) against the oracle, over the sample
    and row by row."""
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, seed=0, weights_device="cuda")
    res = run_gpu(cfg, to_device(inp))
    assert res["err"] == 0
    host = {key: (v.cpu() if isinstance(v, torch.Tensor) else v) for key, v in inp.items()}
    o_idx, _, o_offsets, o_perm = check_routing(cfg, host, res)
    if cfg.T <= 64:
        toks = np.arange(cfg.T)
    else:
        toks = stratified_tokens(o_idx, o_offsets, o_perm, FULL_SAMPLE[name])
        # every routed expert with slots has at least one checked row
        hit = np.unique(o_idx[toks].reshape(-1))
        assert np.array_equal(hit, np.nonzero(np.diff(o_offsets))[0])
    check_outputs(cfg, host, res, tokens=toks)


def test_full_size_shared_experts_separate(cuda_ok):
    """The DeepSeek-V3-shaped layer with its two shared experts run as separate
    groups (the full-size test above runs them merged): a stratified sample of
    tokens against the oracle."""
    cfg = CONFIGS["dsv3"]
    inp = make_inputs(cfg, seed=0, weights_device="cuda")
    res = run_gpu(cfg, to_device(inp), merge_shared=False)
    assert res["err"] == 0
    assert res["y_slots"].shape[0] == cfg.T * (cfg.k + cfg.n_shared)
    host = {key: (v.cpu() if isinstance(v, torch.Tensor) else v) for key, v in inp.items()}
    o_idx, _, o_offsets, o_perm = check_routing(cfg, host, res)
    toks = stratified_tokens(o_idx, o_offsets, o_perm, 512)
    check_outputs(cfg, host, res, tokens=toks)


def test_bounded_wait_expires_and_reports_timeout(cuda_ok):
    """A pipeline wait that nothing satisfies expires, reports MOE_ERR_TIMEOUT
    in the device error word, and leaves the context usable."""
    import ctypes
    import sparse_mixture_experts_07_b200 as moe
    lib = moe.load_library()
    f = lib.moe_selftest_wait_timeout
    f.argtypes = [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert f(0, ctypes.c_void_p(err.data_ptr()), stream) == 1
    assert f(20_000_000, ctypes.c_void_p(err.data_ptr()), stream) == 0
    torch.cuda.synchronize()
    assert err.item() == 1 << 6
    cfg = MoEConfig("after_timeout", T=32, H=128, I=128, E=4, k=2)
    inp, res = _run(cfg)
    assert res["err"] == 0
    check_routing(cfg, inp, res)


def test_token_permutation_permutes_output_rows_exactly(cuda_ok):
    """Each output row depends only on its own token: permuting the tokens
    permutes the rows of y bit for bit (pair kernel, half tiles included)."""
    cfg = MoEConfig("perm_inv", T=1200, H=256, I=192, E=4, k=2, n_shared=1, I_shared=64,
                    routed_scale=2.5)
    inp = make_inputs(cfg)
    a = run_gpu(cfg, to_device(inp))
    pi = torch.from_numpy(np.random.default_rng(0).permutation(cfg.T))
    inp2 = dict(inp)
    inp2["x"] = inp["x"][pi]
    b = run_gpu(cfg, to_device(inp2))
    assert torch.equal(b["topk_idx"], a["topk_idx"][pi])
    assert torch.equal(b["y"], a["y"][pi])


def test_pair_kernel_repeat_runs_are_bit_identical(cuda_ok):
    cfg = MoEConfig("det_pair", T=2048, H=512, I=384, E=8, k=2, zipf_s=1.0)
    inp = to_device(make_inputs(cfg))
    a = run_gpu(cfg, inp)
    b = run_gpu(cfg, inp)
    for key in ("topk_idx", "perm", "y_slots", "y"):
        assert torch.equal(a[key], b[key])


@pytest.mark.parametrize("E,H", [(8, 4096), (40, 200), (64, 2048)])
def test_router_split_planes_sum_to_the_weight(cuda_ok, E, H):
    """hi + mid + lo equals each float32 router weight to within 2^-24 |w|;
    padding rows (experts >= E, rows >= 3 E_PAD) are zero."""
    import sparse_mixture_experts_07_b200 as moe
    shape = moe.Shape(T=512, H=H, I=128, E=E, k=2)
    g = torch.Generator().manual_seed(E)
    w = (torch.randn(E, H, generator=g) * 0.02).cuda()
    ws = moe.router_split(shape, w)
    torch.cuda.synchronize()
    e_pad = next(p for p in (8, 16, 32, 64) if p >= E)
    assert ws.shape == ((3 * e_pad + 15) // 16 * 16, H)
    planes = ws.double().cpu()
    total = planes[:E] + planes[e_pad:e_pad + E] + planes[2 * e_pad:2 * e_pad + E]
    wd = w.double().cpu()
    assert torch.all((total - wd).abs() <= 2.0 ** -24 * wd.abs())
    pad = torch.ones(planes.shape[0], dtype=torch.bool)
    for t in range(3):
        pad[t * e_pad:t * e_pad + E] = False
    assert torch.all(planes[pad] == 0)


@pytest.mark.parametrize("cfg", [
    MoEConfig("split_E8", T=1000, H=512, I=64, E=8, k=2),
    MoEConfig("split_E40_ragged_H", T=700, H=200, I=64, E=40, k=3, zipf_s=1.0),
    MoEConfig("split_E64", T=2100, H=256, I=64, E=64, k=6, zipf_s=1.2),
    MoEConfig("split_k8_E16", T=300, H=4096, I=64, E=16, k=2),
    MoEConfig("split_k4_E64_ragged", T=1000, H=2056, I=64, E=64, k=6, zipf_s=1.2),
], ids=lambda c: c.name)
def test_route_with_presplit_weight_matches_route(cuda_ok, cfg):
    """The router on the weight split at load time (split-K over a cluster
    when the m-tiles leave SMs idle) selects exactly what the router that
    splits the weight in every CTA selects; logits and weights agree within
    the float32 summation bound; repeated calls are bit-identical."""
    import sparse_mixture_experts_07_b200 as moe
    from parity_util import logit_tol
    inp = to_device(make_inputs(cfg))
    shape = moe.Shape.from_config(cfg)
    ws = moe.router_split(shape, inp["w_router"])
    a = moe.route(shape, inp["x"], inp["w_router"], inp["router_bias"], logits=True)
    b = moe.route(shape, inp["x"], inp["w_router"], inp["router_bias"], logits=True, w_split=ws)
    c = moe.route(shape, inp["x"], inp["w_router"], inp["router_bias"], logits=True, w_split=ws)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0])
    tol = logit_tol(cfg.H, a[2].cpu().numpy())
    assert float((a[2] - b[2]).abs().max()) <= tol
    assert float((a[1] - b[1]).abs().max()) <= 2 * tol
    for u, v in zip(b, c):
        assert torch.equal(u, v)


@pytest.mark.parametrize("T,k,E,skew", [
    (1, 1, 4, 0.0),            # one slot
    (700, 1, 256, 0.0),        # E at its maximum, one CTA
    (5001, 3, 64, 1.5),        # cluster of 8, two rounds, ragged last CTA, skewed
    (8192, 2, 8, 0.0),         # the Mixtral-shaped plan: 8 CTAs x one round
    (21845, 3, 16, 0.0),       # 65535 slots: the cluster path's largest plans (8 rounds)
    (65537, 1, 32, 1.0),       # 65537 slots: above it, the three-launch path
    (131073, 2, 64, 1.2),      # 262146 slots over 128 blocks
])
def test_permute_plans_match_the_oracle(cuda_ok, T, k, E, skew):
    """counts, offsets, perm and inv bit-exact against the oracle's counting
    sort, on random expert choices (skewed ones included)."""
    import oracle
    import sparse_mixture_experts_07_b200 as moe
    rng = np.random.default_rng(T)
    p = 1.0 / np.arange(1, E + 1) ** skew
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p / p.sum()) for _ in range(T)]) \
        if T <= 5001 else rng.choice(E, size=(T, k), p=p / p.sum())
    # top-k picks distinct experts per token; the plan itself does not need it
    idx = idx.astype(np.int32)
    shape = moe.Shape(T=T, H=128, I=128, E=E, k=k)
    ws = moe.alloc_workspace(shape)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    counts, offsets, perm, inv = moe.permute(shape, torch.from_numpy(idx).cuda(), ws, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    o_counts, o_offsets, o_perm, o_inv = oracle.permute(idx, E)
    assert np.array_equal(counts.cpu().numpy(), o_counts)
    assert np.array_equal(offsets.cpu().numpy(), o_offsets)
    assert np.array_equal(perm.cpu().numpy(), o_perm)
    assert np.array_equal(inv.cpu().numpy(), o_inv)
