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
    # profiles/traffic_mixtral.md, the capture of this GEMM source (an earlier
    # one read 4.053 GB): gather 0.053 + GEMM 1 2.758 + GEMM 2 1.490 GB
    "mixtral": {"bytes": 4.301e9, "file": "gemm_sm100_pair.cu", "sha": "907865b03f8a6821"},
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


def cpu_oracle_rate_mxfp4(cfg, host_inp, mx_host, budget_s: float = 12.0,
                          max_tokens: int = 4096):
    """Oracle tokens/s of the MXFP4 block (numpy dequantisation of the selected
    experts, then the float64 expert arithmetic) on a bounded token sample."""
    import oracle
    from oracle import mxfp4 as oracle_mx
    oracle.build()
    n = 1
    rng = np.random.default_rng(1)
    while True:
        toks = rng.choice(cfg.T, size=min(n, cfg.T), replace=False)
        t0 = time.perf_counter()
        oracle_mx.moe_block_mxfp4(host_inp["x"], host_inp["w_router"], host_inp["router_bias"],
                                  mx_host["gate_up_q"], mx_host["gate_up_s"], mx_host["down_q"],
                                  mx_host["down_s"], k=cfg.k, routed_scale=cfg.routed_scale,
                                  tokens=toks)
        elapsed = time.perf_counter() - t0
        if elapsed > budget_s / 4 or n >= min(cfg.T, max_tokens):
            break
        n *= 4
    return len(toks) / elapsed, len(toks), elapsed, oracle.threads()


def weights_label(args, cfg) -> str:
    return "mxfp4 (E2M1 codes, E8M0 scales per 32)" if args.weights == "mxfp4" else cfg.dtype


def run_reference(args, cfg, rank, world):
    """The oracle arm: the CPU oracle, as it stands, timed on the host cores on
    bounded token samples of the workload (rank 0 only; other ranks do no work)."""
    if rank != 0:
        return None
    inp = make_inputs(cfg, seed=0, weights_device="cpu")
    mx_host = None
    if args.weights == "mxfp4":
        from sparse_mixture_experts_07_b200.inputs import make_mxfp4_weights
        mx_host = make_mxfp4_weights(cfg, seed=0, device="cpu")

    def rate(budget, max_tokens):
        if mx_host is not None:
            return cpu_oracle_rate_mxfp4(cfg, inp, mx_host, budget_s=budget, max_tokens=max_tokens)
        return cpu_oracle_rate(cfg, inp, budget_s=budget, max_tokens=max_tokens)

    # each step samples tokens for a bounded time, so that K steps stay within
    # about three minutes whatever K is
    step_budget = max(0.2, min(4.0, 180.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        rate(step_budget, 16)
    rates, samples = [], []
    cores = 1
    t_all = time.perf_counter()
    for _ in range(args.steps):
        r, n, el, cores = rate(step_budget, 256)
        rates.append(r)
        samples.append(n)
    wall = time.perf_counter() - t_all
    value = statistics.median(rates)
    what = "the MXFP4 block (numpy dequantisation of the selected experts, float64 expert " \
           "math)" if mx_host is not None else "the block, float64"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * cfg.T / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the named model, random-init weights)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E,
                   "k": cfg.k, "n_shared": cfg.n_shared, "I_shared": cfg.I_shared,
                   "routed_scale": cfg.routed_scale, "weights": weights_label(args, cfg),
                   "storage": cfg.dtype},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {what} for {samples[-1] if samples else 0} "
                                   f"random tokens of the {cfg.T}-token batch (full routing of "
                                   f"those tokens, all their experts); rate per token"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)
    return line


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


def roofline_of(cfg, counts, fwd_ms, region_s, mxfp4, peaks, traffic=None) -> dict:
    """Roofline of the dominant region (moe_forward) from its mean device time.

    Decode batches (T*k <= 256) are HBM-bound: algorithmic bytes (bytes_decode)
    per launch / time, against the measured HBM copy bandwidth.  Prefill is
    tensor-bound: 2*T*(3kHI + 3 S Is H) flops per launch / time, against the
    measured bf16 GEMM throughput (sustained when the timed region is long
    enough to reach the power cap, else the burst figure)."""
    if cfg.T * cfg.k <= 256:
        algo = bytes_decode(cfg, counts, mxfp4=mxfp4)
        achieved = algo / (fwd_ms / 1000.0) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "algorithmic_bytes": algo,
                "kernel": "moe_forward_mxfp4 (activation prep, MXFP4 expert GEMMs and their epilogues)"
                          if mxfp4 else "moe_forward (expert FFN launches)",
                "peak_kind": f"{peaks['source']} HBM copy"}
    flops = 2.0 * cfg.T * (3 * cfg.k * cfg.H * cfg.I + 3 * cfg.n_shared * cfg.I_shared * cfg.H)
    achieved = flops / (fwd_ms / 1000.0) / 1e12
    # a timed region of back-to-back GEMMs longer than ~0.25 s runs into the
    # power cap: compare with the sustained GEMM figure, else the burst one
    long_run = region_s >= 0.25 and peaks["bf16_tflops_sustained"]
    peak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic,
            "kernel": "moe_forward (gather + grouped GEMM gate_up/SwiGLU + grouped GEMM down)",
            "peak_kind": f"{peaks['source']} bf16 {'sustained' if long_run else 'burst'}",
            "frac_of_burst": achieved / peaks["bf16_tflops"]}


class Workload:
    """One configuration on the device: seeded inputs, the layer, its buffers."""

    def __init__(self, cfg, weights: str, dev, seed: int):
        import sparse_mixture_experts_07_b200 as moe
        self.moe = moe
        self.cfg = cfg
        self.inp = make_inputs(cfg, seed=seed, weights_device=str(dev))
        self.shape = moe.Shape.from_config(cfg)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in self.inp.items()}
        self.mx = None
        if weights == "mxfp4":
            from sparse_mixture_experts_07_b200.inputs import make_mxfp4_weights
            self.mx = make_mxfp4_weights(cfg, seed=seed, device=str(dev))
            self.layer = moe.MoELayer(self.shape, d["w_router"], d["router_bias"], mxfp4=self.mx)
        else:
            self.layer = moe.MoELayer(self.shape, d["w_router"], d["router_bias"], d["gate_up"],
                                      d["down"], d["sh_gate_up"], d["sh_down"])
        self.x = d["x"]

    def touched_bytes(self) -> float:
        """Bytes one step must read at least: the active experts' weights for a
        decode batch (from the plan of the last step), all weights otherwise."""
        if self.cfg.T * self.cfg.k <= 256:
            counts = self.layer.buf["counts"].cpu().numpy()
            return bytes_decode(self.cfg, counts, mxfp4=self.mx is not None)
        return float(self.weight_bytes())

    def weight_bytes(self) -> int:
        if self.mx is not None:
            return sum(v.numel() for v in self.mx.values())
        eb = 2 if self.cfg.dtype == "bf16" else 4
        n = self.inp["gate_up"].numel() + self.inp["down"].numel()
        if self.inp["sh_gate_up"] is not None:
            n += self.inp["sh_gate_up"].numel() + self.inp["sh_down"].numel()
        return n * eb

    def forward(self, stream=None):
        """The moe_forward region alone, on the plan the last step left in the buffers."""
        moe, L = self.moe, self.layer
        s = L.shape   # the shape the layer's calls run on (shared experts merged)
        b = L.buf
        if L.mx_prepared is not None:
            moe.forward_mxfp4_prepared(s, self.x, b["offsets"], b["perm"], b["topk_w"], self.mx,
                                       L.mx_prepared, L.workspace, L.err_flag,
                                       y_slots=b["y_slots"], stream=stream)
        elif self.mx is not None:
            moe.forward_mxfp4(s, self.x, b["offsets"], b["perm"], b["topk_w"], self.mx,
                              L.workspace, L.err_flag, y_slots=b["y_slots"], stream=stream)
        else:
            moe.forward(s, self.x, b["offsets"], b["perm"], b["topk_w"], L.gate_up, L.down,
                        L.sh_gate_up, L.sh_down, L.workspace, L.err_flag, y_slots=b["y_slots"],
                        stream=stream)

    def step(self, stream, fwd_start=None, fwd_end=None):
        """route + permute -> forward -> combine, with events around the forward."""
        moe, L = self.moe, self.layer
        s = L.shape
        b = L.buf
        moe.route_permute(s, self.x, L.w_router, L.router_bias, L.workspace, L.err_flag, out=b,
                          stream=stream, w_split=L.w_split)
        if fwd_start is not None:
            fwd_start.record(stream)
        self.forward(stream)
        if fwd_end is not None:
            fwd_end.record(stream)
        moe.combine(s, b["y_slots"], b["inv"], y=b["y"], stream=stream)


# Secondary workloads timed after the headline one in a default run (1 GPU):
# the decode batches (the HBM half of the metric) and the other prefill shapes.
EXTRA_WORKLOADS = [
    ("phimoe_decode1", "bf16"), ("phimoe_decode8", "bf16"), ("phimoe_decode64", "bf16"),
    ("phimoe_decode1", "mxfp4"), ("phimoe_decode8", "mxfp4"), ("phimoe_decode64", "mxfp4"),
    ("gptoss_decode1", "mxfp4"), ("gptoss_decode8", "mxfp4"),
    ("phimoe_prefill", "bf16"), ("gptoss", "bf16"), ("dsv3", "bf16"),
]


def measure_graph(w, stream, steps, flush) -> dict:
    """Decode batches replayed from CUDA graphs: the whole step (MoEGraph, the
    layer's public capture) and the moe_forward region alone, each replay timed
    with CUDA events on `stream`, the L2 flushed first when `flush` is given.
    Without the host's per-launch cost the forward region shows the kernels'
    own device time."""
    step_graph = w.layer.capture(w.x)
    side = torch.cuda.Stream(device=w.x.device)
    side.wait_stream(stream)
    fwd_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(fwd_graph, stream=side):
        w.forward()
    stream.wait_stream(side)
    times = {}
    for key, g in (("ms_per_step", step_graph.graph), ("forward_ms", fwd_graph)):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for _ in range(3):
            g.replay()
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            ev[i][0].record(stream)
            g.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        times[key] = statistics.median(a.elapsed_time(b) for a, b in ev)
    assert w.layer.device_error() == 0, "device error flag set (graph replay)"
    del step_graph, fwd_graph
    return {"graph": {"ms_per_step": times["ms_per_step"],
                      "tokens_per_s": w.cfg.T / (times["ms_per_step"] / 1000.0),
                      "forward_ms": times["forward_ms"]}}


def measure_extra(name, weights, dev, steps, peaks, flush) -> dict:
    """Device time of `steps` steps of one workload, each step timed on its own
    with the L2 flushed in between when the step's weights would fit in L2."""
    cfg = CONFIGS[name]
    w = Workload(cfg, weights, dev, seed=0)
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        w.step(stream)
    torch.cuda.synchronize()
    assert w.layer.device_error() == 0, f"device error flag set ({name})"
    touched = w.touched_bytes()
    need_flush = touched < 4 * L2_BYTES
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        if need_flush:
            flush.zero_()
        e0, e1, f0, f1 = ev[i]
        e0.record(stream)
        w.step(stream, f0, f1)
        e1.record(stream)
    torch.cuda.synchronize()
    assert w.layer.device_error() == 0, f"device error flag set ({name})"
    step_ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    fwd_ms = statistics.median(e[2].elapsed_time(e[3]) for e in ev)
    counts = w.layer.buf["counts"].cpu().numpy()
    roof = roofline_of(cfg, counts, fwd_ms, 0.0, w.mx is not None, peaks)
    keys = ("bound", "achieved", "peak", "unit", "frac", "peak_kind")
    out = {"workload": name, "weights": weights, "T": cfg.T, "steps": steps,
           "ms_per_step": step_ms, "tokens_per_s": cfg.T / (step_ms / 1000.0),
           "forward_ms": fwd_ms, "roofline": {k: roof[k] for k in keys},
           "l2": f"L2 flushed before every step (256 MB write; {touched / 1e9:.3f} GB "
                 "touched per step)" if need_flush
                 else f"weights touched per step {touched / 1e9:.2f} GB > 4x L2, streamed",
           "active_experts": int((counts > 0).sum())}
    if cfg.T * cfg.k <= 256:
        out.update(measure_graph(w, stream, steps, flush if need_flush else None))
        groof = roofline_of(cfg, counts, out["graph"]["forward_ms"], 0.0, w.mx is not None, peaks)
        out["graph"]["roofline"] = {k: groof[k] for k in keys}
    del w
    torch.cuda.empty_cache()
    return out


def measure_train(name, dev, steps, peaks) -> dict:
    """Device time of a training step of the layer: route, plan, the training
    forward (which keeps g, u, h and the gathered x rows), the combine, and
    the backward pass for a fixed upstream gradient.  The roofline counts the
    expert GEMMs: 6 T k H I flops forward and twice that backward (plus the
    shared experts)."""
    import sparse_mixture_experts_07_b200 as moe
    cfg = CONFIGS[name]
    w = Workload(cfg, "bf16", dev, seed=0)
    L, s, x = w.layer, w.layer.shape, w.x
    b = L.buf
    state = torch.empty(moe.train_state_size(s), dtype=torch.uint8, device=dev)
    bws = torch.empty(moe.backward_workspace_size(s), dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev).manual_seed(3)
    dy = torch.randn(cfg.T, cfg.H, generator=g, device=dev).to(torch.bfloat16)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(f0=None, f1=None):
        idx, wt, _ = moe.route(s, x, L.w_router, L.router_bias, out=b, w_split=L.w_split,
                               err_flag=L.err_flag, stream=stream)
        moe.permute(s, idx, L.workspace, L.err_flag, out=b, stream=stream)
        if f0 is not None:
            f0.record(stream)
        moe.forward_train(s, x, b["offsets"], b["perm"], wt, L.gate_up, L.down, L.sh_gate_up,
                          L.sh_down, L.workspace, state, L.err_flag, y_slots=b["y_slots"],
                          stream=stream)
        moe.combine(s, b["y_slots"], b["inv"], y=b["y"], stream=stream)
        moe.backward(s, x, L.w_router, idx, wt, b["counts"], b["offsets"], b["perm"], b["inv"],
                     L.gate_up, L.down, L.sh_gate_up, L.sh_down, state, dy, bws, L.err_flag,
                     logits=logits, aux_coef=0.0, stream=stream)
        if f1 is not None:
            f1.record(stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    assert L.device_error() == 0, f"device error flag set (training {name})"
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for i in range(steps):
        step(ev[i][0], ev[i][1])
    torch.cuda.synchronize()
    assert L.device_error() == 0, f"device error flag set (training {name})"
    ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    fwd_flops = 2.0 * cfg.T * (3 * cfg.k * cfg.H * cfg.I + 3 * cfg.n_shared * cfg.I_shared * cfg.H)
    achieved = 3.0 * fwd_flops / (ms / 1000.0) / 1e12
    out = {"workload": name, "weights": "bf16", "kind": "training step (forward + backward)",
           "T": cfg.T, "steps": steps, "train_ms": ms, "tokens_per_s": cfg.T / (ms / 1000.0),
           "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                        "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                        "peak_kind": f"{peaks['source']} bf16 burst",
                        "region": "training forward + backward of the expert FFNs "
                                  "(flops of the six grouped GEMMs)"}}
    del w, state, bws
    torch.cuda.empty_cache()
    return out


def run_cuda(args, cfg, rank, local, world):
    import sparse_mixture_experts_07_b200 as moe

    dev = torch.device("cuda", local)
    wl = Workload(cfg, args.weights, dev, seed=rank)
    layer, x, mx = wl.layer, wl.x, wl.mx
    stream = torch.cuda.current_stream(dev)

    def step():
        return layer(x)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert layer.device_error() == 0, "device error flag set"

    # ---- device-timed region: K steps, inputs resident in HBM.  When the bytes
    # a step touches would fit in L2 (a small decode batch on MXFP4 weights),
    # the L2 is flushed before every step and the steps are timed one by one.
    n_ev = args.steps
    fwd_start = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    fwd_end = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    b = layer.buf
    touched = wl.touched_bytes()
    flush_l2 = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) \
        if touched < 4 * L2_BYTES else None
    step_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_ev)]
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        s0.record(stream)
        for i in range(args.steps):
            if flush_l2 is not None:
                flush_l2.zero_()
                step_ev[i][0].record(stream)
            wl.step(stream, fwd_start[i], fwd_end[i])
            if flush_l2 is not None:
                step_ev[i][1].record(stream)
        s1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_local = s0.elapsed_time(s1) if flush_l2 is None else \
        sum(e0.elapsed_time(e1) for e0, e1 in step_ev)
    del flush_l2
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
    tr = TRAFFIC.get(cfg.name)
    traffic = None
    if tr and mx is None:
        src = os.path.join(ROOT, "sparse_mixture_experts_07_b200", "csrc", tr["file"])
        if os.path.exists(src) and tr.get("sha") == src_sha(src):
            traffic = tr["bytes"]
    roof = roofline_of(cfg, counts, fwd_ms, ms_total / 1000.0, mx is not None, peaks, traffic)
    roof.pop("algorithmic_bytes", None)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f16" if mx is not None else ("bf16" if cfg.dtype == "bf16" else "f32"),
        "data": "synthetic (seeded; shapes of the named model, random-init weights)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E,
                   "k": cfg.k, "n_shared": cfg.n_shared, "I_shared": cfg.I_shared,
                   "routed_scale": cfg.routed_scale, "weights": weights_label(args, cfg),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "L2 flushed before every step (its touched bytes, "
                         f"{touched / 1e9:.3f} GB, would fit in 4x L2); steps timed one by one"
                         if touched < 4 * L2_BYTES else
                         "inputs larger than L2 (expert weights touched per step "
                         f"{touched / 1e9:.2f} GB, streamed every step)"},
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
        host = host_inputs(wl.inp)
        hm = {k: v.cpu() for k, v in mx.items()}
        r, n, el, cores = cpu_oracle_rate_mxfp4(cfg, host, hm)
        line["cpu_baseline"] = {
            "value": r, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"the MXFP4 block for {n} of the {cfg.T} tokens ({el:.1f} s: numpy "
                      "dequantisation of the selected experts, then float64 expert math)"}
    elif rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = host_inputs(wl.inp)
        r, n, el, cores = cpu_oracle_rate(cfg, host)
        line["cpu_baseline"] = {
            "value": r, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"the block for {n} random tokens of the {cfg.T}-token batch "
                      f"({el:.1f} s, float64, OpenMP over tokens); rate per token"}
    del layer, wl, x_host, y_host, x_dev, y_dev
    torch.cuda.empty_cache()

    # ---- the other workloads (1 GPU only): decode batches and prefill shapes,
    # each with the roofline fraction of its forward
    if world == 1 and not args.no_extra:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        extra = []
        with ClockSampler(local) as clk2:
            for name, weights in EXTRA_WORKLOADS:
                if name == cfg.name and weights == args.weights:
                    continue
                extra.append(measure_extra(name, weights, dev, max(10, min(args.steps, 50)),
                                           peaks, flush))
            if not args.no_train:
                extra.append(measure_train("mixtral", dev, max(5, min(args.steps, 20)), peaks))
        line["workloads"] = extra
        line["workloads_clocks"] = clk2.summary()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="mixtral", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the headline workload (skip the decode and prefill lines)")
    ap.add_argument("--no-train", action="store_true",
                    help="skip the training-step line among the extra workloads")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "mxfp4"],
                    help="expert weight format; mxfp4 runs the decode path (T <= 64)")
    args = ap.parse_args()
    cfg = CONFIGS[args.config]
    if args.weights == "mxfp4" and not (cfg.T <= 64 and cfg.dtype == "bf16" and cfg.n_shared == 0):
        ap.error("--weights mxfp4 needs a bf16 decode configuration (T <= 64, no shared experts)")
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
