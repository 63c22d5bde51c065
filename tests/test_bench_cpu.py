"""The host arithmetic of bench.py on the CPU: the algorithmic bytes and FLOPs behind the
roofline fraction, the choice of the binding roofline, and the oracle's timed CPU leg."""
import numpy as np
import pytest

import bench
from nvfp4_mixture_experts_w4a4_b200 import workloads as W

PEAKS = {"hbm_gbs": 6532.9, "fp4_tflops": 4 * 1618.8}


def test_decode_gate_up_bytes_by_hand():
    """Decode (T16 H2048 I512 k10) with 140 touched experts: each expert's gate and up weights
    once (2 x 512 x 2048 elements at 4.5 bits), the x codes and scales of the 160 permuted rows,
    and their h codes and scales written once."""
    wl = W.WORKLOADS["decode"]
    alg = bench.algorithmic(wl, n_active=140, gemm_path=True)
    w13 = 140 * 1_179_648           # 2*512*2048 * 0.5625 bytes per expert
    x_rows = 160 * 2048 * 9 // 16   # 1152 bytes per permuted row
    h_rows = 160 * 512 * 9 // 16    # 288 bytes per permuted row
    assert alg["gate_up_bytes"] == w13 + x_rows + h_rows == 165_381_120
    assert alg["gate_up_flops"] == 2.0 * 160 * 2 * 2048 * 512
    assert alg["flops"] == 2.0 * 160 * 3 * 2048 * 512


def test_gemv_path_reads_x_once_per_token_and_a16_in_bf16():
    wl = W.WORKLOADS["decode"]
    tc = bench.algorithmic(wl, 100, gemm_path=True)
    gv = bench.algorithmic(wl, 100, gemm_path=False)
    a16 = bench.algorithmic(wl, 100, gemm_path=False, a16=True)
    assert tc["gate_up_bytes"] - gv["gate_up_bytes"] == (160 - 16) * 2048 * 0.5625
    # bf16 x per token and bf16 h per row instead of 0.5625 bytes per element
    assert a16["gate_up_bytes"] - gv["gate_up_bytes"] == 16 * 2048 * (2 - 0.5625) + 160 * 512 * (2 - 0.5625)


def test_shared_expert_adds_to_the_layer_not_to_gate_up():
    wl = W.WORKLOADS["decode"]
    base = bench.algorithmic(wl, 140, True)
    sh = bench.algorithmic(wl, 140, True, shared_I=512)
    assert sh["gate_up_bytes"] == base["gate_up_bytes"]
    assert sh["layer_bytes"] - base["layer_bytes"] == 3 * 2048 * 512 * 2
    assert sh["flops"] - base["flops"] == 2.0 * 16 * 3 * 2048 * 512


def test_roofline_picks_the_binding_resource():
    # 165 MB in 37 us is bandwidth-bound: its FLOPs take far less time at the FP4 peak
    r = bench.roofline(165_381_120, 671_088_640, 0.037, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(165_381_120 / 37e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6532.9)
    assert r["nominal"] == {"peak": 8000.0, "frac": pytest.approx(r["achieved"] / 8000.0)}
    # the dense 512-token gate/up: 2*512*2*5120*17408 FLOPs over about 200 MB is compute-bound
    wl = W.WORKLOADS["dense"]
    alg = bench.algorithmic(wl, 1, True)
    r = bench.roofline(alg["gate_up_bytes"], alg["gate_up_flops"], 0.0615, PEAKS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["frac"] == pytest.approx(alg["gate_up_flops"] / 61.5e-6 / 1e12 / PEAKS["fp4_tflops"])
    assert r["nominal"]["peak"] == 9000.0 and r["nominal"]["frac"] == pytest.approx(r["achieved"] / 9000.0)


@pytest.mark.parametrize("a16", [False, True])
def test_oracle_leg_runs_on_the_cpu(a16):
    """The cpu_baseline leg times the oracle alone: seeded inputs drawn on the host, the
    oracle's own weight quantisation and (W4A4) its own per-expert h calibration."""
    wl = W.WORKLOADS["tiny"]
    rate, threads, sample = bench.oracle_rate(wl, budget_s=0.5, max_tokens=4, a16=a16)
    assert rate > 0 and threads >= 1
    assert sample.startswith("4 of 8 tokens per pass")
    assert np.isfinite(rate)
    r1, t1, _ = bench.oracle_rate(wl, budget_s=0.2, max_tokens=4, a16=a16, nthreads=1)
    assert t1 == 1 and r1 > 0


def test_reference_arm_never_loads_the_gpu_library():
    """bench.py --impl reference: the oracle on host-drawn inputs; libnvfp4moe.so is never
    mapped into the process (checked in a fresh interpreter)."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import argparse, bench\n"
        "from nvfp4_mixture_experts_w4a4_b200 import workloads as W\n"
        "bench.reference_arm(argparse.Namespace(steps=1, warmup=1, act='nvfp4'), W.WORKLOADS['tiny'], 0, 1, False)\n"
        "maps = open('/proc/self/maps').read()\n"
        "print('MAPPED' if 'libnvfp4moe' in maps else 'NOT_MAPPED')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    out = r.stdout.strip().splitlines()
    assert out[-1] == "NOT_MAPPED"
    line = json.loads(out[-2])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["cores"] >= 1 and "cpu_model" in line["cpu_baseline"]


def test_oracle_inputs_draw_only_the_sampled_tokens_experts():
    import oracle as O
    wl = W.WORKLOADS["decode"]
    x, logits, arr, s_x = bench.oracle_inputs(wl, 2)
    ids, _ = O.route(logits, wl.k)
    used = set(np.unique(ids).tolist())
    sc = arr["g"][2]
    assert {int(e) for e in np.nonzero(sc != 1.0)[0]} <= used
    assert all(sc[e] != 1.0 for e in used)  # every used expert was quantised (tensor scale set)
    assert x.shape == (2, wl.H) and s_x > 0
