"""bench.py host logic on the CPU: the oracle arm (`--impl reference`) prints
one parseable JSON line on rank 0, for bf16/float32 and for MXFP4 weights, and
the roofline helper counts the algorithmic work of each regime."""
import argparse
import json
import os
import subprocess
import sys

import numpy as np

import bench
from sparse_mixture_experts_07_b200.inputs import CONFIGS, MoEConfig

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line_from_the_command_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny" and d["config"]["weights"] == "f32"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_times_the_mxfp4_oracle_for_mxfp4_weights(capsys):
    cfg = MoEConfig("mx_bench", T=4, H=64, I=64, E=4, k=2)
    args = argparse.Namespace(steps=2, warmup=1, weights="mxfp4")
    line = bench.run_reference(args, cfg, rank=0, world=1)
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1 and json.loads(out[0]) == json.loads(json.dumps(line))
    assert line["config"]["weights"].startswith("mxfp4")
    assert "MXFP4" in line["cpu_baseline"]["sample"]
    assert line["value"] > 0


def test_roofline_regimes():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1300.0,
             "source": "test"}
    dec = CONFIGS["phimoe_decode1"]
    counts = np.zeros(dec.E, dtype=np.int32)
    counts[[3, 7]] = 1
    r = bench.roofline_of(dec, counts, fwd_ms=0.1, region_s=0.0, mxfp4=False, peaks=peaks)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == bench.bytes_decode(dec, counts) / 1e-4 / 1e9
    assert r["frac"] == r["achieved"] / 6000.0
    pre = CONFIGS["dsv3"]
    r = bench.roofline_of(pre, None, fwd_ms=2.0, region_s=0.1, mxfp4=False, peaks=peaks)
    flops = 2.0 * pre.T * (3 * pre.k * pre.H * pre.I + 3 * 2 * 1024 * pre.H)
    assert r["bound"] == "tensor" and r["peak"] == 1600.0
    assert abs(r["achieved"] - flops / 2e-3 / 1e12) < 1e-9
    r = bench.roofline_of(pre, None, fwd_ms=2.0, region_s=0.5, mxfp4=False, peaks=peaks)
    assert r["peak"] == 1300.0 and "sustained" in r["peak_kind"]


def test_extra_workloads_are_known_configurations():
    for name, weights in bench.EXTRA_WORKLOADS:
        cfg = CONFIGS[name]
        assert weights in ("bf16", "mxfp4")
        if weights == "mxfp4":
            assert cfg.T <= 64 and cfg.n_shared == 0
