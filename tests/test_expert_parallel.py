"""Expert parallelism: the partition of the experts, the all-reduce of the
ranks' partial outputs, and the per-rank CUDA pieces.

CPU: the split of E experts over N ranks; two gloo ranks that each compute
the oracle's partial for their experts and sum them with the same
allreduce_partial the GPU path uses, against the whole block.
GPU (one device): N ranks emulated one after another on the same GPU, each
running moe_forward_experts and moe_combine_experts on its own experts'
weights; their float32 partials are summed (standing in for the all-reduce)
and rounded by moe_cast_f32, against the oracle and the one-rank layer.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_mixture_experts_07_b200.expert_parallel import expert_range
from sparse_mixture_experts_07_b200.inputs import MoEConfig, make_inputs


@pytest.mark.parametrize("E,world", [(8, 1), (8, 2), (8, 3), (64, 8), (16, 5), (2, 4)])
def test_expert_ranges_cover_the_experts_once(E, world):
    ranges = [expert_range(E, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == E
    for (a0, b0), (a1, b1) in zip(ranges[:-1], ranges[1:]):
        assert b0 == a1
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == E
    assert sizes == sorted(sizes, reverse=True)


def test_expert_range_rejects_bad_ranks():
    for args in ((8, 0, 0), (8, 2, 2), (8, 2, -1)):
        with pytest.raises(ValueError):
            expert_range(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


EP_CPU_CFG = MoEConfig("ep_cpu", T=12, H=16, I=8, E=6, k=2, n_shared=1, I_shared=4,
                       routed_scale=2.5, dtype="f32", zipf_s=1.0)


def _gloo_rank(rank, world, port, outdir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    import datetime

    import torch.distributed as dist

    import oracle
    from sparse_mixture_experts_07_b200.expert_parallel import allreduce_partial
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    cfg = EP_CPU_CFG
    inp = make_inputs(cfg, seed=0)
    a, b = expert_range(cfg.E, world, rank)
    part = oracle.moe_block_experts(inp, k=cfg.k, routed_scale=cfg.routed_scale, e_begin=a,
                                    e_end=b, with_shared=(rank == 0))
    t = torch.from_numpy(part)
    allreduce_partial(t)
    np.save(os.path.join(outdir, f"y{rank}.npy"), t.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_sum_their_expert_partials_to_the_block(tmp_path):
    import oracle
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_gloo_rank, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    cfg = EP_CPU_CFG
    y, _, _ = oracle.moe_block(make_inputs(cfg, seed=0), k=cfg.k, routed_scale=cfg.routed_scale)
    for r in range(world):
        yr = np.load(tmp_path / f"y{r}.npy")
        assert np.linalg.norm(yr - y) <= 1e-13 * np.linalg.norm(y)


# ------------------------------------------------------------------- GPU
EP_GPU = [
    (MoEConfig("ep_bf16_shared", T=700, H=256, I=192, E=8, k=2, n_shared=2, I_shared=128,
               routed_scale=2.5, zipf_s=1.0), 3),
    (MoEConfig("ep_bf16_pair", T=2048, H=384, I=256, E=8, k=2), 2),
    (MoEConfig("ep_bf16_many", T=512, H=256, I=136, E=64, k=6, n_shared=2, I_shared=128,
               routed_scale=2.5, zipf_s=1.2), 8),
    (MoEConfig("ep_decode", T=7, H=512, I=256, E=16, k=2, n_shared=1, I_shared=128), 4),
    (MoEConfig("ep_f32", T=90, H=64, I=96, E=6, k=3, dtype="f32", zipf_s=1.0), 4),
    (MoEConfig("ep_more_ranks_than_k", T=300, H=128, I=128, E=4, k=2), 4),
]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg,world", EP_GPU, ids=lambda v: getattr(v, "name", str(v)))
def test_emulated_ranks_match_the_oracle_and_one_rank(cuda_ok, cfg, world):
    import oracle
    import sparse_mixture_experts_07_b200 as moe
    from parity_util import check_outputs, rel_l2, to_device
    inp = make_inputs(cfg, seed=0)
    d = to_device(inp)
    shape = moe.Shape.from_config(cfg)
    # shared experts as separate groups, like the ranks' layers (slot rows compared)
    full = moe.MoELayer(shape, d["w_router"], d["router_bias"], d["gate_up"], d["down"],
                        d["sh_gate_up"], d["sh_down"], merge_shared=False)
    y_full = full(d["x"]).clone()
    slots_full = full.last["y_slots"].clone()
    offsets = full.last["offsets"].cpu().numpy()
    total = torch.zeros(cfg.T, cfg.H, dtype=torch.float32, device="cuda")
    for r in range(world):
        a, b = expert_range(cfg.E, world, r)
        layer = moe.MoELayerEP(shape, r, world, d["w_router"], d["router_bias"],
                               d["gate_up"][a:b].contiguous(), d["down"][a:b].contiguous(),
                               d["sh_gate_up"], d["sh_down"])
        part = layer.partial(d["x"])
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        # the rank's slot rows are those of the one-rank forward, bit for bit
        lo, hi = int(offsets[a]), int(offsets[b])
        assert torch.equal(layer.buf["y_slots"][lo:hi], slots_full[lo:hi])
        if r == 0 and cfg.n_shared:
            tk = cfg.T * cfg.k
            assert torch.equal(layer.buf["y_slots"][tk:], slots_full[tk:])
        total += part
    y = moe.cast_f32(shape, total)
    torch.cuda.synchronize()
    res = {"y": y.cpu()}
    check_outputs(cfg, inp, res)
    assert rel_l2(y.float().cpu().numpy().astype(np.float64),
                  y_full.float().cpu().numpy().astype(np.float64)) <= 1e-3
    # the partial of each rank alone equals the oracle's partial
    a, b = expert_range(cfg.E, world, world - 1)
    last = moe.MoELayerEP(shape, world - 1, world, d["w_router"], d["router_bias"],
                          d["gate_up"][a:b].contiguous(), d["down"][a:b].contiguous())
    part = last.partial(d["x"]).cpu().numpy().astype(np.float64)
    ref = oracle.moe_block_experts(inp, k=cfg.k, routed_scale=cfg.routed_scale, e_begin=a,
                                   e_end=b, with_shared=False)
    if np.linalg.norm(ref) > 0:
        assert rel_l2(part, ref) <= (1e-2 if cfg.dtype == "bf16" else 1e-5)
