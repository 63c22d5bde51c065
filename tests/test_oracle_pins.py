"""Pins for the CPU oracle: checks it against things other than itself.

* the format's own tables, through ml_dtypes (a third-party E2M1 / E4M3 implementation),
  torch's float8_e4m3fn, and the CUDA toolkit headers' host conversions;
* hand-worked 16-element blocks (tests/golden/quant_blocks.json);
* round-trips of every representable block, saturation, zero and underflow blocks;
* an independent numpy/ml_dtypes quantiser on random data, bit for bit;
* the exact block GEMM against a brute-force fp64 dequantise-then-matmul;
* top-k against a sort, softmax-over-k against a renormalised full softmax;
* the permutation against counting-sort invariants;
* the whole layer against a direct per-token formulation that never permutes.
"""
import json
import os
import shutil
import subprocess

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import refquant as R

HERE = os.path.dirname(os.path.abspath(__file__))
F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def _tie_points():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    mids = [(a + b) / 2 for a, b in zip(grid, grid[1:])]
    pts = []
    for m in mids + grid + [6.5, 7.0, 100.0, 1e30]:
        f = np.float32(m)
        pts += [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))]
    pts = np.array(pts, np.float32)
    return np.concatenate([pts, -pts])


# ------------------------------------------------------------------ E2M1 ----
def test_e2m1_table_exhaustive_vs_ml_dtypes():
    ref = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    got = np.array([O.e2m1_value(c) for c in range(16)])
    assert np.array_equal(np.signbit(got), np.signbit(ref))
    assert np.array_equal(got, ref)
    # magnitudes are the NVFP4 grid
    assert list(got[:8]) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_encode_vs_ml_dtypes():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        _tie_points(),
        rng.uniform(-8, 8, 200_000).astype(np.float32),
        rng.standard_normal(50_000).astype(np.float32) * np.float32(3),
        np.float32([0.0, -0.0, 1e-30, -1e-30, 0.2499999, -0.2500001]),
    ])
    got = O.e2m1_encode_array(vals)
    ref = R.e2m1_codes_from_values(vals)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (vals[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_e2m1_tie_table():
    # ties go to the even code; saturation above 6; the sign survives rounding to zero
    cases = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 6.5: 7, 1e9: 7,
             -0.1: 8, -0.25: 8, -5.0: 14}
    for v, c in cases.items():
        assert O.e2m1_encode(v) == c, v


# ------------------------------------------------------------------ E4M3 ----
def test_e4m3_table_exhaustive_vs_ml_dtypes_and_torch():
    ref = np.arange(256, dtype=np.uint8).view(F8).astype(np.float64)
    ref_t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([O.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(got[~nan], ref_t[~nan])
    assert O.e4m3_value(0x7E) == 448.0 and O.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_encode_vs_ml_dtypes_and_torch():
    rng = np.random.default_rng(2)
    finite = np.arange(256, dtype=np.uint8).view(F8).astype(np.float32)
    finite = finite[np.isfinite(finite)]
    mids = ((finite[:-1].astype(np.float64) + finite[1:]) / 2).astype(np.float32)
    vals = np.concatenate([
        finite, mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(-np.inf)),
        np.exp(rng.uniform(np.log(1e-4), np.log(448), 200_000)).astype(np.float32),
    ])
    vals = np.concatenate([vals, -vals])
    vals = vals[np.abs(vals) <= 448]
    got = O.e4m3_encode_array(vals)
    ref = R.e4m3_codes_from_values(vals)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (vals[bad[:5]], got[bad[:5]], ref[bad[:5]])
    ref_t = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref_t)


def test_e4m3_saturates_to_finite():
    for v in [448.0, 449.0, 464.0, 465.0, 1e6, 3e38]:
        assert O.e4m3_encode(v) == 0x7E
        assert O.e4m3_encode(-v) == 0xFE


def test_finite_e4m3_roundtrip():
    for c in range(0, 0x7F):
        assert O.e4m3_encode(O.e4m3_value(c)) == c
        assert O.e4m3_encode(-O.e4m3_value(c)) == (c | 0x80)


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.exists("/usr/local/cuda/include/cuda_fp4.h"),
                    reason="needs g++ and the CUDA toolkit headers")
def test_codecs_vs_cuda_header_host_conversions(tmp_path):
    exe = tmp_path / "conv"
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I/usr/local/cuda/include",
                           os.path.join(HERE, "helpers", "cuda_header_conv.cpp"), "-o", str(exe)])
    rng = np.random.default_rng(3)
    vals = np.concatenate([
        _tie_points(), rng.uniform(-8, 8, 100_000).astype(np.float32),
        np.exp(rng.uniform(np.log(1e-4), np.log(600), 100_000)).astype(np.float32),
    ]).astype(np.float32)
    out = subprocess.run([str(exe)], input=vals.tobytes(), capture_output=True, check=True).stdout
    out = np.frombuffer(out, np.uint8).reshape(-1, 2)
    assert np.array_equal(O.e2m1_encode_array(vals), out[:, 0])
    assert np.array_equal(O.e4m3_encode_array(vals), out[:, 1])


# ------------------------------------------------------------- quantiser ----
def _golden_blocks():
    with open(os.path.join(HERE, "golden", "quant_blocks.json")) as f:
        return json.load(f)["blocks"]


@pytest.mark.parametrize("blk", _golden_blocks(), ids=lambda b: b["name"])
def test_hand_worked_blocks(blk):
    x = np.array([float(v) for v in blk["x"]], np.float32)[None, :]
    s_t = float(np.float32(float(blk["s_t"])))
    codes, sf, ts = O.quantize(x, tensor_scale=s_t)
    assert sf[0, 0] == int(blk["sf"], 16)
    assert list(codes[0]) == [int(b, 16) for b in blk["bytes"]]
    unpacked = [(codes[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(16)]
    assert unpacked == blk["codes"]


def test_roundtrip_every_block_scale():
    # a block holding every code (so its amax is 6) times every non-zero finite block
    # scale quantises back to the same scale and codes with s_t = 1
    codes16 = np.arange(16, dtype=np.uint8)
    vals = codes16.view(F4).astype(np.float32)
    for sfc in range(1, 0x7F):
        sfv = np.float32(np.uint8(sfc).view(F8).astype(np.float32))
        x = (vals * sfv).astype(np.float32)[None, :]
        c, s, _ = O.quantize(x, tensor_scale=1.0)
        assert s[0, 0] == sfc
        unpacked = np.stack([c[0] & 0xF, c[0] >> 4], 1).ravel()
        assert np.array_equal(unpacked, codes16), sfc


def test_dynamic_tensor_scale():
    x = np.zeros((2, 32), np.float32)
    x[1, 5] = -5376.0  # amax 5376 = 2 * 2688
    _, _, ts = O.quantize(x)
    assert ts == 2.0
    x = np.zeros((3, 16), np.float32)
    c, s, ts = O.quantize(x)
    assert ts == 0.0 and not c.any() and not s.any()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_quantiser_vs_independent_numpy_formulation(seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    x[:, rng.choice(512, 5, replace=False)] *= 20  # outlier channels
    x[3, :16] = 0  # a zero block
    x[7, 16:32] *= 1e-6  # an underflowing block
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    for given in [None, 1e-3, 0.7]:
        c, s, ts = O.quantize(x, tensor_scale=given)
        if given is None:
            assert ts == np.float32(np.abs(x).max()) / np.float32(2688)
        rc, rs = R.quantize(x, np.float32(ts))
        assert np.array_equal(s, rs)
        assert np.array_equal(c, rc)


def test_dequantize_vs_ml_dtypes():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    c, s, ts = O.quantize(x)
    assert np.array_equal(O.dequantize(c, s, ts), R.dequantize(c, s, ts))
    # quantisation error is bounded by half a grid step of the largest magnitude (<=1/3
    # relative to the block amax) plus the scale rounding
    err = np.abs(O.dequantize(c, s, ts) - x)
    amax = np.abs(x.reshape(8, 4, 16)).max(2)
    assert (err.reshape(8, 4, 16).max(2) <= amax * 0.35).all()


# ------------------------------------------------------------------ GEMM ----
@pytest.mark.parametrize("shape", [(1, 1, 16), (3, 5, 48), (7, 9, 256), (16, 33, 64)])
def test_block_gemm_vs_fp64_bruteforce(shape):
    M, N, K = shape
    rng = np.random.default_rng(M * 100 + N)
    a = rng.standard_normal((M, K)).astype(np.float32) * 3
    b = rng.standard_normal((N, K)).astype(np.float32) / np.sqrt(K)
    ac, asf, sa = O.quantize(a)
    bc, bsf, sb = O.quantize(b)
    got = O.gemm(ac, asf, sa, bc, bsf, sb, nthreads=2)
    ref = R.dequantize(ac, asf, sa) @ R.dequantize(bc, bsf, sb).T
    scale = np.abs(R.dequantize(ac, asf, sa)) @ np.abs(R.dequantize(bc, bsf, sb)).T + 1e-300
    assert (np.abs(got - ref) <= 1e-13 * scale).all()
    # a transposed operand or a dropped block would be caught
    if M == N and M > 1:
        assert not np.allclose(got, got.T)


# ------------------------------------------------------------- routing ----
def _ref_topk(logits, k):
    T, E = logits.shape
    ids = np.zeros((T, k), np.int32)
    for t in range(T):
        # sort by descending logit, ties by ascending index (+0 and -0 compare equal)
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))
        ids[t] = order[:k]
    return ids


def test_route_vs_sort_and_full_softmax():
    rng = np.random.default_rng(7)
    T, E, k = 50, 64, 6
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[0, :] = 0.5  # all tied
    logits[1, ::2] = 0.0
    logits[1, 1::2] = -0.0  # +0 / -0 ties
    logits[2, 10] = logits[2, 20] = logits[2, 30] = 9.0
    ids, w = O.route(logits, k)
    assert np.array_equal(ids, _ref_topk(logits, k))
    assert list(ids[0]) == list(range(k))
    assert list(ids[2, :3]) == [10, 20, 30]
    # softmax over the k selected == full softmax renormalised over them
    full = np.exp(logits.astype(np.float64) - logits.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    sel = np.take_along_axis(full, ids.astype(np.int64), 1)
    np.testing.assert_allclose(w, sel / sel.sum(1, keepdims=True), rtol=2e-7, atol=0)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-6)


def test_route_k_equals_e_and_e1():
    logits = np.array([[1.0, 3.0, 2.0]], np.float32)
    ids, w = O.route(logits, 3)
    assert list(ids[0]) == [1, 2, 0]
    ids, w = O.route(np.zeros((4, 1), np.float32), 1)
    assert (ids == 0).all() and (w == 1.0).all()


# ----------------------------------------------------------- permutation ----
def test_permute_invariants():
    rng = np.random.default_rng(9)
    T, E, k = 37, 16, 4
    ids, _ = O.route(rng.standard_normal((T, E)).astype(np.float32), k)
    p = O.permute(ids, E)
    assert np.array_equal(p["counts"], np.bincount(ids.ravel(), minlength=E))
    assert np.array_equal(p["offsets"], np.concatenate([[0], np.cumsum(p["counts"])]))
    pairs = np.arange(T * k)
    rows = p["pair_to_row"]
    assert np.array_equal(np.sort(rows), pairs)  # a bijection
    assert np.array_equal(p["row_token"][rows], pairs // k)
    assert np.array_equal(p["row_slot"][rows], pairs % k)
    for e in range(E):
        seg = slice(p["offsets"][e], p["offsets"][e + 1])
        toks = p["row_token"][seg]
        assert (np.diff(toks) > 0).all()  # stable: ascending token order
        assert (ids[toks, p["row_slot"][seg]] == e).all()
    with pytest.raises(ValueError):
        O.permute(np.array([[0, 16]], np.int32), E)


# ------------------------------------------------------------- the layer ----
def _tiny_layer_inputs(T=8, H=256, I=128, E=8, k=2, seed=0):
    from nvfp4_mixture_experts_w4a4_b200 import workloads as W
    wl = W.scaled(W.WORKLOADS["tiny"], T=T, H=H, I=I, E=E, k=k)
    act = W.make_activations(wl, seed)
    wts = W.make_weights(wl, seed)
    x = act["x"].view(torch.int16).numpy().view(np.uint16)
    logits = act["logits"].numpy()
    wg = O.quantize_experts(wts["w_gate"].numpy())
    wu = O.quantize_experts(wts["w_up"].numpy())
    wd = O.quantize_experts(wts["w_down"].numpy())
    return wl, x, logits, wg, wu, wd


def _direct_layer(x_bf16, logits, k, wg, wu, wd, s_h):
    """Per-token, per-slot formulation: no permutation, dequantise-then-matmul in fp64,
    the quantiser taken from the independent numpy/ml_dtypes formulation."""
    xf = x_bf16.view(np.uint16).astype(np.uint32) << 16
    xf = xf.view(np.float32)
    T, H = xf.shape
    s_x = np.float32(np.abs(xf).max()) / np.float32(2688)
    xc, xs = R.quantize(xf, s_x)
    xdq = R.dequantize(xc, xs, s_x)
    ids = _ref_topk(logits, k)
    out = np.zeros((T, H))
    for t in range(T):
        sel = logits[t, ids[t]].astype(np.float64)
        wts = np.exp(sel - sel[0])
        wts = (wts / wts.sum()).astype(np.float32).astype(np.float64)
        for j in range(k):
            e = ids[t, j]
            g = R.dequantize(wg[0][e], wg[1][e], wg[2][e]) @ xdq[t]
            u = R.dequantize(wu[0][e], wu[1][e], wu[2][e]) @ xdq[t]
            h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
            hc, hs = R.quantize(h[None, :], np.float32(s_h[e]))
            y = R.dequantize(wd[0][e], wd[1][e], wd[2][e]) @ R.dequantize(hc, hs, s_h[e])[0]
            out[t] += wts[j] * y
    return out


def test_layer_vs_direct_per_token_formulation():
    wl, x, logits, wg, wu, wd = _tiny_layer_inputs()
    r = O.moe_ffn(x, logits, wl.k, wg, wu, wd, nthreads=2)
    ref = _direct_layer(x, logits, wl.k, wg, wu, wd, r["h_scale"])
    assert np.abs(r["out_f64"] - ref).max() <= 1e-9 * np.abs(ref).max()
    # bf16 output is the round-to-nearest-even of the fp32 rounding of out_f64
    f32 = r["out_f64"].astype(np.float32)
    assert np.array_equal(r["out_bf16"], torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    # calibrated per-expert requant scales are amax(h)/2688 over each expert's rows
    for e in range(wl.E):
        seg = slice(r["offsets"][e], r["offsets"][e + 1])
        if r["counts"][e]:
            assert r["h_scale"][e] == np.float32(np.abs(r["h_f32"][seg]).max()) / np.float32(2688)


def test_layer_given_scales_and_dense_special_case():
    wl, x, logits, wg, wu, wd = _tiny_layer_inputs(T=5, E=1, k=1)
    s_h = np.full(1, 0.01, np.float32)
    r = O.moe_ffn(x, np.zeros((5, 1), np.float32), 1, wg, wu, wd, x_scale=0.002, h_scale=s_h)
    assert r["x_scale"] == np.float32(0.002)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    xc, xs = R.quantize(xf, np.float32(0.002))
    assert np.array_equal(r["x_codes"], xc) and np.array_equal(r["x_sf"], xs)
    # dense: y = W_d . q(silu(W_g x) * (W_u x)), no weights
    xdq = R.dequantize(xc, xs, np.float32(0.002))
    g = xdq @ R.dequantize(wg[0][0], wg[1][0], wg[2][0]).T
    u = xdq @ R.dequantize(wu[0][0], wu[1][0], wu[2][0]).T
    h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
    hc, hs = R.quantize(h, np.float32(0.01))
    assert np.array_equal(r["h_codes"], hc) and np.array_equal(r["h_sf"], hs)
    y = R.dequantize(hc, hs, np.float32(0.01)) @ R.dequantize(wd[0][0], wd[1][0], wd[2][0]).T
    assert np.abs(r["out_f64"] - y).max() <= 1e-9 * np.abs(y).max()


def test_layer_expert_with_no_tokens_and_all_tokens_one_expert():
    wl, x, logits, wg, wu, wd = _tiny_layer_inputs(T=6, E=4, k=1)
    logits = np.full((6, 4), -1.0, np.float32)
    logits[:, 2] = 1.0  # everyone picks expert 2
    r = O.moe_ffn(x, logits, 1, wg, wu, wd)
    assert list(r["counts"]) == [0, 0, 6, 0]
    assert list(r["row_token"]) == list(range(6))
    assert (r["w"] == 1.0).all()
    assert r["h_scale"][0] == 1.0 and r["h_scale"][2] > 0


@pytest.mark.parametrize("seed", [1, 2])
def test_layer_invariant_under_expert_relabeling(seed):
    """Experts have no order of their own: relabeling them (permuting the logit columns and the
    weight stacks together) must leave routing, combine weights and the output bit-for-bit
    unchanged, while the permuted rows follow the new labels.  A mix-up of expert indices
    anywhere (weights, per-expert scales, counts, offsets) breaks it."""
    wl, x, logits, wg, wu, wd = _tiny_layer_inputs()
    p = np.random.default_rng(seed).permutation(wl.E)  # new expert i is old expert p[i]
    relabel = lambda w: tuple(np.ascontiguousarray(a[p]) for a in w)  # noqa: E731
    r0 = O.moe_ffn(x, logits, wl.k, wg, wu, wd, nthreads=2)
    r1 = O.moe_ffn(x, np.ascontiguousarray(logits[:, p]), wl.k, relabel(wg), relabel(wu), relabel(wd), nthreads=2)
    assert np.array_equal(p[r1["ids"]], r0["ids"])
    assert np.array_equal(r1["w"], r0["w"])
    assert np.array_equal(r1["counts"], r0["counts"][p])
    assert np.array_equal(r1["h_scale"], r0["h_scale"][p])
    assert np.array_equal(r1["out_bf16"], r0["out_bf16"])
    assert np.array_equal(r1["out_f64"], r0["out_f64"])
    # the same pair lands in a row of its expert's new segment, with the same h codes
    for t in range(wl.T):
        for j in range(wl.k):
            a, b_ = r0["pair_to_row"][t * wl.k + j], r1["pair_to_row"][t * wl.k + j]
            assert np.array_equal(r0["h_codes"][a], r1["h_codes"][b_])


@pytest.mark.parametrize("w4a16", [False, True])
def test_layer_equivariant_under_token_reordering(w4a16):
    """Tokens are independent apart from the shared scales (the x tensor scale and the per-
    expert h scales, maxima that ignore order): reordering the tokens reorders the output rows
    and changes nothing else.  A mix-up of token and row indices breaks it."""
    wl, x, logits, wg, wu, wd = _tiny_layer_inputs()
    q = np.random.default_rng(5).permutation(wl.T)
    run = O.moe_ffn_w4a16 if w4a16 else O.moe_ffn
    r0 = run(x, logits, wl.k, wg, wu, wd, nthreads=2)
    r1 = run(np.ascontiguousarray(x[q]), np.ascontiguousarray(logits[q]), wl.k, wg, wu, wd, nthreads=2)
    assert np.array_equal(r1["ids"], r0["ids"][q])
    assert np.array_equal(r1["out_bf16"], r0["out_bf16"][q])
    assert np.array_equal(r1["out_f64"], r0["out_f64"][q])
    if not w4a16:
        assert np.array_equal(r1["h_scale"], r0["h_scale"]) and r1["x_scale"] == r0["x_scale"]


# ------------------------------------------------------- weight-only layer ----
def _bf16_round(a):
    """fp64 -> fp32 -> bf16 (round to nearest even at each step, by torch), as float64."""
    t = torch.from_numpy(np.asarray(a, np.float64).astype(np.float32)).to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def test_w4a16_layer_vs_direct_per_token_formulation():
    """Weight-only variant against a per-token formulation: no permutation, weights
    dequantised by the independent ml_dtypes formulation, fp64 matmuls, h rounded to bf16
    by torch."""
    wl, x, logits, wg, wu, wd = _tiny_layer_inputs(T=7, E=6, k=3)
    r = O.moe_ffn_w4a16(x, logits, wl.k, wg, wu, wd, nthreads=2)
    xf = ((x.astype(np.uint32) << 16).view(np.float32)).astype(np.float64)
    ids = _ref_topk(logits, wl.k)
    assert np.array_equal(r["ids"], ids)
    ref = np.zeros((wl.T, wl.H))
    for t in range(wl.T):
        sel = logits[t, ids[t]].astype(np.float64)
        wts = np.exp(sel - sel[0])
        wts = (wts / wts.sum()).astype(np.float32).astype(np.float64)
        for j in range(wl.k):
            e = ids[t, j]
            g = R.dequantize(wg[0][e], wg[1][e], wg[2][e]) @ xf[t]
            u = R.dequantize(wu[0][e], wu[1][e], wu[2][e]) @ xf[t]
            h = _bf16_round(g / (1 + np.exp(-g)) * u)
            ref[t] += wts[j] * (R.dequantize(wd[0][e], wd[1][e], wd[2][e]) @ h)
            row = r["pair_to_row"][t * wl.k + j]
            hb = (r["h_bf16"][row].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            # h is bf16(fp32(silu(g) u)); the fp64 sums may differ in the last bits, so a
            # rounding boundary may fall either way: at most one bf16 step apart
            assert np.all(np.abs(hb - h) <= np.abs(h) * 2.0 ** -7 + 1e-30)
    assert np.abs(r["out_f64"] - ref).max() <= 1e-6 * np.abs(ref).max()


def test_w4a16_identity_experts_closed_form():
    """Experts whose NVFP4 weights encode identities (gate = up = I, down = c_e I): the layer
    reduces to out[t][n] = sum_j w_tj c_{e_tj} bf16(silu(x_tn) x_tn), written out here
    with math.exp."""
    import math
    T, H, E, k = 5, 16, 4, 2
    I = H
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    xf = x.to(torch.float64).numpy()
    logits = rng.standard_normal((T, E)).astype(np.float32)
    codes = np.zeros((E, I, H // 2), np.uint8)
    for i in range(I):  # E2M1 code 2 is 1.0; element i sits in byte i // 2, nibble i % 2
        codes[:, i, i // 2] = 2 << (4 * (i % 2))
    sf = np.full((E, I, H // 16), 0x38, np.uint8)  # E4M3 0x38 is 1.0
    ones = np.ones(E, np.float32)
    c = np.array([0.5, 1.0, 2.0, 0.25], np.float32)
    r = O.moe_ffn_w4a16(xb, logits, k, (codes, sf, ones), (codes, sf, ones), (codes, sf, c))
    ids = _ref_topk(logits, k)
    for t in range(T):
        sel = [float(logits[t, e]) for e in ids[t]]
        ex = [math.exp(v - sel[0]) for v in sel]
        wts = [float(np.float32(v / sum(ex))) for v in ex]
        for n in range(H):
            h = float(_bf16_round(xf[t, n] / (1 + math.exp(-xf[t, n])) * xf[t, n]))
            want = sum(wts[j] * float(c[ids[t, j]]) * h for j in range(k))
            assert abs(r["out_f64"][t, n] - want) <= 1e-6 * max(abs(want), 1e-30), (t, n)


# -------------------------------------------------------------------- MXFP4 ----
def test_e8m0_table_vs_ml_dtypes():
    F80 = ml_dtypes.float8_e8m0fnu
    for c in range(256):
        ref = float(np.array([c], np.uint8).view(F80)[0])
        got = O.e8m0_value(c)
        assert (np.isnan(ref) and np.isnan(got)) or ref == got, c


def _mx_golden():
    with open(os.path.join(HERE, "golden", "mx_blocks.json")) as f:
        return json.load(f)["blocks"]


@pytest.mark.parametrize("blk", _mx_golden(), ids=lambda b: b["name"])
def test_mx_hand_worked_blocks(blk):
    x = np.array(blk["x"], np.float32)[None, :]
    codes, e8m0 = O.mx_quantize(x)
    assert int(e8m0[0, 0]) == blk["e8m0"]
    unpacked = [(int(codes[0, i // 2]) >> (4 * (i % 2))) & 0xF for i in range(32)]
    assert unpacked == blk["codes"]


def test_mx_quantiser_vs_numpy_formulation():
    """MX quantisation written with numpy (frexp for the exponent) and ml_dtypes' E2M1 cast,
    bit for bit on random blocks of several magnitudes."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((24, 128)) * np.exp2(rng.integers(-20, 20, (24, 1)))).astype(np.float32)
    x[3, :32] = 0.0
    codes, e8m0 = O.mx_quantize(x)
    blocks = x.reshape(24, 4, 32).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    _, e = np.frexp(amax)
    X = np.where(amax > 0, np.clip(e - 3, -127, 127), -127)
    assert np.array_equal(e8m0, (X + 127).astype(np.uint8))
    q = np.clip(blocks / np.exp2(X)[..., None], -6.0, 6.0).astype(np.float32)
    ref = q.astype(F4).view(np.uint8).reshape(24, 128) & 0xF
    got = np.stack([(codes >> 0) & 0xF, codes >> 4], axis=2).reshape(24, 128)
    assert np.array_equal(got, ref)


def test_mx_roundtrip_of_representable_blocks():
    """A block built from E2M1 values times one power of two comes back exactly."""
    rng = np.random.default_rng(12)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    vals = grid[rng.integers(0, 8, (16, 64))] * np.where(rng.random((16, 64)) < 0.5, -1, 1)
    vals[:, ::32] = 6.0  # pin each block's largest magnitude to 6 so X is the power chosen below
    p = np.exp2(rng.integers(-30, 30, (16, 2)).repeat(32, axis=1))
    x = (vals * p).astype(np.float32)
    codes, e8m0 = O.mx_quantize(x)
    assert np.array_equal(O.mx_dequantize(codes, e8m0), x.astype(np.float64))


def test_mx_to_nvfp4_is_exact_and_refuses_wide_spans():
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((32, 256)) * np.exp2(rng.integers(-8, 9, (32, 1)))).astype(np.float32)
    codes, e8m0 = O.mx_quantize(x)
    c2, sf, ts = O.mx_to_nvfp4(codes, e8m0)
    assert np.array_equal(c2, codes)
    assert np.array_equal(O.dequantize(codes, sf, ts), O.mx_dequantize(codes, e8m0))
    # 2^-20 next to 2^0 spans more than the 18 binades of E4M3 powers of two
    y = np.ones((2, 64), np.float32)
    y[1, :32] = 2.0 ** -20
    c, e = O.mx_quantize(y)
    with pytest.raises(ValueError):
        O.mx_to_nvfp4(c, e)


# ------------------------------------------------------------- shared expert ----
def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_shared_expert_identity_closed_form():
    """Shared expert with identity gate/up and down = c * I (bf16, exact): the layer output moves
    by exactly c * bf16(silu(x) x) per element (math.exp), with the routed part unchanged."""
    import math
    wl, x, logits, wg, wu, wd = _tiny_layer_inputs(T=4, H=256, I=128, E=4, k=2)
    H = wl.H
    eye = np.eye(H, dtype=np.float32)
    c = 0.75
    shared = (_bf16_bits(eye), _bf16_bits(eye), _bf16_bits(c * eye))
    r0 = O.moe_ffn(x, logits, wl.k, wg, wu, wd, nthreads=2)
    r1 = O.moe_ffn(x, logits, wl.k, wg, wu, wd, h_scale=r0["h_scale"], x_scale=r0["x_scale"], shared=shared,
                   nthreads=2)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(wl.T):
        for n in range(H):
            v = xf[t, n]
            want = c * float(_bf16_round(v / (1 + math.exp(-v)) * v))
            assert abs((r1["out_f64"][t, n] - r0["out_f64"][t, n]) - want) <= 1e-9 * max(1.0, abs(want))
    # the weight-only layer adds the same term
    a0 = O.moe_ffn_w4a16(x, logits, wl.k, wg, wu, wd, nthreads=2)
    a1 = O.moe_ffn_w4a16(x, logits, wl.k, wg, wu, wd, shared=shared, nthreads=2)
    assert np.allclose(a1["out_f64"] - a0["out_f64"], r1["out_f64"] - r0["out_f64"], rtol=0, atol=1e-9)


def test_shared_expert_vs_numpy_formulation():
    """Random bf16 shared weights: the added term equals Wd . bf16(silu(Wg x) (Wu x)) written with
    numpy matmuls and torch's bf16 rounding."""
    rng = np.random.default_rng(21)
    wl, x, logits, wg, wu, wd = _tiny_layer_inputs(T=5, H=256, I=128, E=4, k=2)
    Is = 64
    g = rng.standard_normal((Is, wl.H)) / 16
    u = rng.standard_normal((Is, wl.H)) / 16
    d = rng.standard_normal((wl.H, Is)) / 8
    shared = (_bf16_bits(g), _bf16_bits(u), _bf16_bits(d))
    back = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)  # noqa: E731
    r0 = O.moe_ffn(x, logits, wl.k, wg, wu, wd, nthreads=2)
    r1 = O.moe_ffn(x, logits, wl.k, wg, wu, wd, h_scale=r0["h_scale"], x_scale=r0["x_scale"], shared=shared,
                   nthreads=2)
    xf = back(x)
    gv = xf @ back(shared[0]).T
    uv = xf @ back(shared[1]).T
    h = _bf16_round(gv / (1 + np.exp(-gv)) * uv)
    ys = h @ back(shared[2]).T
    assert np.abs((r1["out_f64"] - r0["out_f64"]) - ys).max() <= 1e-9 * np.abs(ys).max()
