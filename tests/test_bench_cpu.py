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
    """The cpu_baseline leg times the oracle alone: seeded inputs, the oracle's own weight
    quantisation and (W4A4) its own per-expert h calibration."""
    wl = W.WORKLOADS["tiny"]
    act = W.make_activations(wl, 0, "cpu")
    wts = W.make_weights(wl, 0, "cpu")
    host = {e: {n: wts[n][e].numpy() for n in ("w_gate", "w_up", "w_down")} for e in range(wl.E)}
    rate, threads, sample = bench.oracle_rate(wl, act, host, None, budget_s=0.5, max_tokens=4, a16=a16)
    assert rate > 0 and threads >= 1
    assert sample.startswith("4 of 8 tokens per pass")
    assert np.isfinite(rate)
