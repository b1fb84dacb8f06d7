"""Benchmark of the dropless sparse MoE feed-forward block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

One step = the whole block (route -> permute -> expert FFNs -> combine) over
one batch of T synthetic tokens, inputs resident in HBM.  The default workload
is the Mixtral-8x7B-shaped layer (T=4096, H=4096, I=14336, E=8, k=2, bf16).
Prints one JSON line (rank 0).  Under torchrun every rank runs an independent
replica on its own tokens (no data-path collective: weak scaling).

`--impl reference` times the CPU oracle (the plain reference implementation of
the block) on the host cores, on bounded token samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_07_b200.inputs import CONFIGS, make_inputs  # noqa: E402

METRIC = "moe_layer_tokens_per_s"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024

# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant
# kernels, from one ncu capture, keyed by workload; valid only while the GEMM
# source is unchanged (sha256 of the file, first 16 hex digits).
TRAFFIC = {
    # profiles/grouped_gemm_pair_mixtral.md: gather 0.053 + GEMM 1 3.410 + GEMM 2 1.687 GB
    "mixtral": {"bytes": 5.149e9, "file": "gemm_sm100_pair.cu", "sha": "1ef98e621b42032d"},
}


def src_sha(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        loaded = [v for v in sm if v > 0.5 * max(sm)]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, local, world


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_rate(cfg, host_inp, budget_s: float = 12.0, max_tokens: int = 4096):
    """Oracle tokens/s on a bounded token sample (grown until ~budget_s/4 per try)."""
    import oracle
    oracle.build()
    n, elapsed = 4, 0.0
    rng = np.random.default_rng(1)
    while True:
        toks = rng.choice(cfg.T, size=min(n, cfg.T), replace=False)
        t0 = time.perf_counter()
        oracle.moe_block(host_inp, k=cfg.k, routed_scale=cfg.routed_scale, tokens=toks)
        elapsed = time.perf_counter() - t0
        if elapsed > budget_s / 4 or n >= min(cfg.T, max_tokens):
            break
        n *= 4
    return len(toks) / elapsed, len(toks), elapsed, oracle.threads()


def host_inputs(inp: dict) -> dict:
    return {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def bytes_decode(cfg, counts, mxfp4: bool = False) -> float:
    """Algorithmic HBM bytes of one decode step: the touched experts' weights
    once (MXFP4: half a byte per weight plus one scale byte per 32), the router
    weight, x in, y out, and the slot buffer written and read."""
    eb = 2 if cfg.dtype == "bf16" else 4
    wb = 0.5 + 1.0 / 32.0 if mxfp4 else eb
    active = int((counts > 0).sum())
    w = active * 3 * cfg.H * cfg.I * wb + cfg.n_shared * 3 * cfg.H * cfg.I_shared * eb
    return w + cfg.E * cfg.H * 4 + 2 * cfg.T * cfg.H * eb + \
        2 * cfg.T * (cfg.k + cfg.n_shared) * cfg.H * eb


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return
    inp = make_inputs(cfg, seed=0, weights_device="cpu")
    # each step samples tokens for a bounded time, so that K steps stay within
    # about three minutes whatever K is
    step_budget = max(0.2, min(4.0, 180.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_rate(cfg, inp, budget_s=step_budget, max_tokens=16)
    rates, samples = [], []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        r, n, el, cores = cpu_oracle_rate(cfg, inp, budget_s=step_budget, max_tokens=256)
        rates.append(r)
        samples.append(n)
    wall = time.perf_counter() - t_all
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * cfg.T / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the named model, random-init weights)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E,
                   "k": cfg.k, "n_shared": cfg.n_shared, "I_shared": cfg.I_shared,
                   "routed_scale": cfg.routed_scale,
                   "weights": "mxfp4 (E2M1 codes, E8M0 scales per 32)" if mx is not None
                              else cfg.dtype, "storage": cfg.dtype},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: the block for {samples[-1]} random tokens of the "
                                   f"{cfg.T}-token batch (full routing of those tokens, all their "
                                   f"experts), float64; rate extrapolated per token"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)


def count_launches(step_fn) -> int:
    """Kernels of libmoe.so launched by one step (CUPTI via torch.profiler)."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    try:
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step_fn()
            torch.cuda.synchronize()
    except Exception:       # CUPTI unavailable (e.g. under another profiler)
        return -1
    n = 0
    for ev in prof.events():
        name = ev.name or ""
        if ev.device_type.name == "CUDA" and "moe::" in name:
            n += 1
    return n


def run_cuda(args, cfg, rank, local, world):
    import sparse_mixture_experts_07_b200 as moe

    dev = torch.device("cuda", local)
    inp = make_inputs(cfg, seed=rank, weights_device=str(dev))
    shape = moe.Shape.from_config(cfg)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    mx = None
    if args.weights == "mxfp4":
        from sparse_mixture_experts_07_b200.inputs import make_mxfp4_weights
        mx = make_mxfp4_weights(cfg, seed=rank, device=str(dev))
        layer = moe.MoELayer(shape, d["w_router"], d["router_bias"], mxfp4=mx)
    else:
        layer = moe.MoELayer(shape, d["w_router"], d["router_bias"], d["gate_up"], d["down"],
                             d["sh_gate_up"], d["sh_down"])
    x = d["x"]
    stream = torch.cuda.current_stream(dev)

    def step():
        return layer(x)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert layer.device_error() == 0, "device error flag set"

    # ---- device-timed region: K steps, inputs resident in HBM
    n_ev = args.steps
    fwd_start = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    fwd_end = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    b = layer.buf
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        s0.record(stream)
        for i in range(args.steps):
            idx, w, _ = moe.route(shape, x, layer.w_router, layer.router_bias, out=b,
                                  w_split=layer.w_split,
                                  err_flag=layer.err_flag)
            moe.permute(shape, idx, layer.workspace, layer.err_flag, out=b)
            fwd_start[i].record(stream)
            if mx is not None:
                moe.forward_mxfp4(shape, x, b["offsets"], b["perm"], w, mx, layer.workspace,
                                  layer.err_flag, y_slots=b["y_slots"])
            else:
                moe.forward(shape, x, b["offsets"], b["perm"], w, layer.gate_up, layer.down,
                            layer.sh_gate_up, layer.sh_down, layer.workspace, layer.err_flag,
                            y_slots=b["y_slots"])
            fwd_end[i].record(stream)
            moe.combine(shape, b["y_slots"], b["inv"], y=b["y"])
        s1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_local = s0.elapsed_time(s1)
    fwd_ms = statistics.mean(fwd_start[i].elapsed_time(fwd_end[i]) for i in range(n_ev))
    ms_total = max_over_ranks(ms_local, world)
    tokens = cfg.T * args.steps * world
    value = tokens / (ms_total / 1000.0)
    counts = b["counts"].cpu().numpy()

    # ---- end to end through the public API with host buffers: every step copies
    # its x in from pinned host memory and its y back out, pipelined the way a
    # serving loop runs: the copy-in of step i+1 and the copy-out of step i-1
    # run on their own streams while step i computes (double-buffered x and y).
    x_host = [x.cpu().pin_memory() for _ in range(2)]
    y_host = [torch.empty(cfg.T, cfg.H, dtype=x.dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    y_dev = [torch.empty_like(b["y"]) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    copied_in = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    copied_out = [torch.cuda.Event() for _ in range(2)]
    x_free = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n_steps, t0=None, t1=None):
        for i in range(n_steps):
            j = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(x_free[j])            # step i-2 done reading x_dev[j]
                if i == 0 and t0 is not None:
                    t0.record(s_in)
                x_dev[j].copy_(x_host[j], non_blocking=True)
                copied_in[j].record(s_in)
            stream.wait_event(copied_in[j])
            if i >= 2:
                stream.wait_event(copied_out[j])          # y_dev[j] drained by step i-2
            layer(x_dev[j], stream=stream, y=y_dev[j])
            x_free[j].record(stream)
            computed[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[j])
                y_host[j].copy_(y_dev[j], non_blocking=True)
                copied_out[j].record(s_out)
        if t1 is not None:
            t1.record(s_out)

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_run(3)
    barrier(world)
    torch.cuda.synchronize()
    e2e_run(args.steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = tokens / (e2e_ms / 1000.0)
    assert torch.equal(y_host[(args.steps - 1) & 1], y_dev[(args.steps - 1) & 1].cpu())
    eb = 2 if cfg.dtype == "bf16" else 4

    launches_per_step = count_launches(step)
    assert layer.device_error() == 0, "device error flag set"

    peaks = measured_peaks()
    decode = cfg.T * cfg.k <= 256
    tr = TRAFFIC.get(cfg.name)
    traffic = None
    if tr:
        src = os.path.join(ROOT, "sparse_mixture_experts_07_b200", "csrc", tr["file"])
        if os.path.exists(src) and tr.get("sha") == src_sha(src):
            traffic = tr["bytes"]
    if decode:
        algo = bytes_decode(cfg, counts, mxfp4=mx is not None)
        achieved = algo / (fwd_ms / 1000.0) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "kernel": "moe_forward_mxfp4 (f16 prep + MXFP4 expert FFN launches)"
                          if mx is not None else "moe_forward (expert FFN launches)",
                "peak_kind": f"{peaks['source']} HBM copy"}
    else:
        flops = 2.0 * cfg.T * (3 * cfg.k * cfg.H * cfg.I + 3 * cfg.n_shared * cfg.I_shared * cfg.H)
        achieved = flops / (fwd_ms / 1000.0) / 1e12
        # a timed region of back-to-back GEMMs longer than ~0.25 s runs into the
        # power cap: compare with the sustained GEMM figure, else the burst one
        long_run = ms_total / 1000.0 >= 0.25 and peaks["bf16_tflops_sustained"]
        peak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "kernel": "moe_forward (gather + grouped GEMM gate_up/SwiGLU + grouped GEMM down)",
                "peak_kind": f"{peaks['source']} bf16 {'sustained' if long_run else 'burst'}",
                "frac_of_burst": achieved / peaks["bf16_tflops"]}

    if mx is not None:
        weight_bytes = sum(v.numel() for v in mx.values())
    else:
        weight_bytes = (inp["gate_up"].numel() + inp["down"].numel()) * eb
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f16" if mx is not None else ("bf16" if cfg.dtype == "bf16" else "f32"),
        "data": "synthetic (seeded; shapes of the named model, random-init weights)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E,
                   "k": cfg.k, "n_shared": cfg.n_shared, "I_shared": cfg.I_shared,
                   "routed_scale": cfg.routed_scale,
                   "weights": "mxfp4 (E2M1 codes, E8M0 scales per 32)" if mx is not None
                              else cfg.dtype,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (expert weights "
                         f"{weight_bytes / 1e9:.2f} GB streamed every step)"},
        "tflops": 2.0 * cfg.T * (cfg.H * cfg.E + 3 * cfg.k * cfg.H * cfg.I +
                                 3 * cfg.n_shared * cfg.I_shared * cfg.H) * args.steps * world /
                  (ms_total / 1000.0) / 1e12,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": cfg.T * cfg.H * eb,
                "d2h_bytes_per_step": cfg.T * cfg.H * eb},
        "gpu_launches": launches_per_step * args.steps if launches_per_step >= 0 else None,
        "clocks": clk.summary(),
        "expert_counts": counts.tolist(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and mx is not None:
        # the oracle's MXFP4 block on the whole (decode) batch: dequantise the
        # selected experts, then the float64 expert math
        import oracle
        from oracle import mxfp4 as oracle_mx
        host = host_inputs(inp)
        hm = {k: v.cpu() for k, v in mx.items()}
        t0 = time.perf_counter()
        oracle_mx.moe_block_mxfp4(host["x"], host["w_router"], host["router_bias"],
                                  hm["gate_up_q"], hm["gate_up_s"], hm["down_q"], hm["down_s"],
                                  k=cfg.k, routed_scale=cfg.routed_scale)
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {
            "value": cfg.T / el, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"the MXFP4 block for all {cfg.T} tokens ({el:.1f} s: numpy dequantisation "
                      "of the selected experts, then float64 expert math)"}
    elif rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = host_inputs(inp)
        r, n, el, cores = cpu_oracle_rate(cfg, host)
        line["cpu_baseline"] = {
            "value": r, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"the block for {n} random tokens of the {cfg.T}-token batch "
                      f"({el:.1f} s, float64, OpenMP over tokens); rate per token"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del layer


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="mixtral", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "mxfp4"],
                    help="expert weight format; mxfp4 runs the decode path (T <= 8)")
    args = ap.parse_args()
    cfg = CONFIGS[args.config]
    if args.weights == "mxfp4" and not (cfg.T <= 8 and cfg.dtype == "bf16" and cfg.n_shared == 0):
        ap.error("--weights mxfp4 needs a bf16 decode configuration (T <= 8, no shared experts)")
    rank, local, world = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, cfg, rank, world)
        else:
            run_cuda(args, cfg, rank, local, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
