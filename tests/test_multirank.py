"""The N>1 host path of bench.py (replicas; no data-path collective), run as
two gloo ranks on the CPU: process-group set-up from the torchrun
environment, the barrier, and the max-over-ranks timing reduction."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    import torch.distributed as dist
    r, local, w = bench.dist_setup()
    bench.barrier(w)
    # each rank reports its own device time; the job time is the slowest rank's
    ms = bench.max_over_ranks(10.0 + 5.0 * r, w)
    tokens = 4096 * 3 * w           # T per replica x steps x ranks
    with open(os.path.join(outdir, f"rank{r}.json"), "w") as f:
        json.dump({"rank": r, "world": w, "ms": ms, "tokens_per_s": tokens / (ms / 1000.0),
                   "backend": dist.get_backend()}, f)
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for d in res:
        assert d["world"] == 2 and d["backend"] == "gloo"
        assert d["ms"] == 15.0
        assert d["tokens_per_s"] == pytest.approx(4096 * 3 * 2 / 0.015)


def test_reference_arm_other_ranks_do_no_work(capsys):
    import argparse

    import bench
    from sparse_mixture_experts_07_b200.inputs import CONFIGS
    args = argparse.Namespace(steps=1, warmup=0)
    bench.run_reference(args, CONFIGS["tiny"], rank=1, world=2)
    assert capsys.readouterr().out == ""
