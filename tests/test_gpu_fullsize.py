"""Parity at the full sizes the benchmark times (gpu): every token of the decode-sized
batches, and at least 64 chosen tokens of the larger ones.

The library runs each workload's whole batch on the device with the benchmark's settings
(dynamic x scale, path chosen automatically, seeded draws of workloads.py).  The oracle
computes, from the same fp32 weights and bf16 inputs and without anything from the device:
  * the routing of every token and the permutation (bit-exact against the device's);
  * the layer input's tensor scale over the whole batch (bit-exact);
  * the NVFP4 codes of every expert the sampled tokens use (bit-exact against the device's
    quantised weights);
  * the checked tokens' x codes, h codes and outputs, with per-expert h scales that it
    calibrates on them and that the device then uses too.
Decode (16 tokens) and dense T=1 are checked whole.  Prefill chunk, long prefill and dense
T=512 check at least 64 tokens: the first and last token of every 192-row chunk (the wide
tiling's token tile) of the experts with the most tokens, the first and last token of the
batch, and tokens spread evenly over the rest, so that every late tile, ragged chunk tail
and accumulator of the largest groups is read at least once.
The oracle runs the sample with only the experts the sample uses: a token's top-k over a set
of experts that contains its own top-k is the same top-k in the same order, so restricting the
logits to those columns changes neither the selection nor the weights."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_mixture_experts_w4a4_b200 import _lib as C
from nvfp4_mixture_experts_w4a4_b200 import ops, workloads as W
from tests import gpu_util as G
from tests.helpers import layouts as LY
from tests.helpers import refquant as R

pytestmark = pytest.mark.gpu

MIN_SAMPLE = 64  # tokens checked at least, when the batch is larger than that
CHUNK = 192      # token rows per tile of the wide tiling (batches above 64 tokens)


def checked_tokens(ids_all: np.ndarray, T: int, E: int) -> np.ndarray:
    """Every token when T <= 64; otherwise the chunk-boundary tokens of the largest experts,
    the batch's first and last token, and MIN_SAMPLE evenly spread tokens."""
    if T <= MIN_SAMPLE:
        return np.arange(T)
    perm = O.permute(ids_all, E)
    counts, offsets, row_token = perm["counts"], perm["offsets"], perm["row_token"]
    sel = {0, T - 1}
    for e in np.argsort(-counts, kind="stable")[:6]:
        rows = row_token[offsets[e]:offsets[e + 1]]
        for c0 in range(0, len(rows), CHUNK):
            sel.add(int(rows[c0]))
            sel.add(int(rows[min(c0 + CHUNK, len(rows)) - 1]))
    sel.update(int(t_) for t_ in np.linspace(0, T - 1, MIN_SAMPLE).round().astype(np.int64))
    return np.array(sorted(sel), np.int64)


@pytest.mark.parametrize("name,shared_I,launch", [
    ("decode", 0, "auto"), ("prefill_chunk", 0, "auto"), ("long_prefill", 0, "auto"), ("dense", 0, "auto"),
    ("dense_t1", 0, "auto"), ("decode", 512, "auto"), ("prefill_chunk", 512, "auto"),
    ("decode", 0, "single_local"), ("decode", 0, "single_tile"), ("decode", 0, "multi")])
def test_fullsize_sampled_tokens(name, shared_I, launch):
    """shared_I > 0: with a BF16 shared expert of that size (the streamed kernel at 16 tokens,
    the tcgen05 bf16 GEMMs at 512).  launch: the automatic choice (as the benchmark runs it), or
    the decode batch forced through each single-launch schedule and the multi-launch path."""
    wl = W.WORKLOADS[name]
    dev = G.need_gpu()
    T, H, I, E, k = wl.T, wl.H, wl.I, wl.E, wl.k
    act = W.make_activations(wl, 0, dev)
    wts = W.make_weights(wl, 0, dev)
    experts = ops.NVFP4Experts.from_float(wts["w_gate"], wts["w_up"], wts["w_down"])
    torch.cuda.synchronize()

    x_bits = G.bf16_bits(act["x"])
    logits = act["logits"].cpu().numpy()
    # oracle: routing of the whole batch, permutation, the layer input's tensor scale
    ids_all, w_all = O.route(logits, k)
    sample = checked_tokens(ids_all, T, E)
    perm = O.permute(ids_all, E)
    _, _, s_x = O.quantize(G.bits_to_f32(x_bits))
    touched = np.unique(ids_all[sample])

    # oracle quantisation of the touched experts, checked against the device's codes
    tt = torch.as_tensor(touched, device=dev)
    wg = G.quantize_experts_parallel(wts["w_gate"][tt].cpu().numpy())
    wu = G.quantize_experts_parallel(wts["w_up"][tt].cpu().numpy())
    wd = G.quantize_experts_parallel(wts["w_down"][tt].cpu().numpy())
    del wts
    ref_w = LY.experts_to_device_layout(wg, wu, wd)
    got_w = [experts.w13_codes, experts.w13_sf, experts.w13_scale, experts.w2_codes, experts.w2_sf,
             experts.w2_scale]
    for r, g in zip(ref_w, got_w):
        assert np.array_equal(g[tt].cpu().numpy(), r)

    # oracle on the sample, restricted to the touched experts; it calibrates s_h on the sample
    shared, shared_bits = None, None
    if shared_I:
        gate, up, down, shared_bits = G.shared_weights(wl, shared_I)
        shared = (ops.shared_expert_w13(gate.to(dev), up.to(dev)), down.to(dev))
    ref = O.moe_ffn(x_bits[sample], logits[sample][:, touched], k, wg, wu, wd, x_scale=s_x, shared=shared_bits)
    assert np.array_equal(touched[ref["ids"]], ids_all[sample])
    s_h = np.ones(E, np.float32)
    s_h[touched] = ref["h_scale"]

    # the device: the whole batch, dynamic x scale, automatic path
    mode = {"auto": C.LAUNCH_AUTO, "single_local": C.LAUNCH_SINGLE_LOCAL, "single_tile": C.LAUNCH_SINGLE_TILE,
            "multi": C.LAUNCH_MULTI}[launch]
    layer = ops.MoeFFN(experts, k, torch.from_numpy(s_h).to(dev), shared=shared, launch=mode)
    if launch != "auto":
        assert layer.layout(T).single_launch == (0 if launch == "multi" else 1)
    out = layer(act["x"], act["logits"])
    torch.cuda.synchronize()
    im = layer.intermediates(T)

    # routing and permutation of the whole batch: bit-exact
    assert np.array_equal(im["topk_ids"].cpu().numpy(), ids_all)
    np.testing.assert_allclose(im["topk_w"].cpu().numpy(), w_all, rtol=2e-6, atol=1e-7)
    assert np.array_equal(im["counts"].cpu().numpy(), perm["counts"])
    assert np.array_equal(im["offsets"].cpu().numpy(), perm["offsets"])
    p2r = im["pair_to_row"].cpu().numpy()
    po = im["padded_offsets"].cpu().numpy()
    e_of_pair = ids_all.reshape(-1)
    assert np.array_equal(p2r - po[e_of_pair] + perm["offsets"][e_of_pair], perm["pair_to_row"])
    # x scale: bit-exact
    assert im["x_scale"].item() == np.float32(s_x)

    # sampled pairs: x codes bit-exact, h codes within the requantisation tolerance
    gpu_pairs = (sample[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    ref_pairs = np.arange(len(sample) * k)
    gpu_rows = p2r[gpu_pairs]
    ref_rows = ref["pair_to_row"][ref_pairs]
    x_rows = gpu_rows if im["path"] == C.PATH_GEMM else np.repeat(sample, k)
    xc = im["x_codes"].cpu().numpy()[x_rows]
    xsf = LY.from_mma(im["x_sf"].cpu().numpy(), im["x_rows"], H)[x_rows]
    tok = np.repeat(np.arange(len(sample)), k)
    assert np.array_equal(xc, ref["x_codes"][tok])
    assert np.array_equal(xsf, ref["x_sf"][tok])
    hc_pairs = im["h_codes"].cpu().numpy()[gpu_rows]
    hsf_pairs = LY.from_mma(im["h_sf"].cpu().numpy(), im["h_rows"], I)[gpu_rows]
    # reorder into the oracle's row order
    order = np.argsort(ref_rows)
    hc = np.empty_like(hc_pairs)
    hsf = np.empty_like(hsf_pairs)
    hc[ref_rows[order]] = hc_pairs[order]
    hsf[ref_rows[order]] = hsf_pairs[order]
    n_diff = G.check_h_codes(hc, hsf, ref["h_codes"], ref["h_sf"])

    # sampled outputs within the stated tolerance (widened by the first-order effect of any
    # allowed h code difference)
    extra = None
    if n_diff:
        wl_s = W.scaled(wl, T=len(sample), E=len(touched))
        extra = G.h_diff_effect(hc, hsf, ref, wl_s, lambda e: R.dequantize(wd[0][e], wd[1][e], wd[2][e]))
    print(f"[full size] {name}: {len(sample)} tokens, {len(touched)} experts, {n_diff} h codes differ")
    G.check_out(G.bf16_bits(out)[sample], ref["out_f64"], extra=extra)


@pytest.mark.parametrize("name", ["decode", "dense_t1"])
def test_fullsize_weight_only_sampled_tokens(name):
    """The weight-only (W4A16) variant at full size, as the benchmark runs it with --act bf16:
    routing and permutation of the whole batch bit-exact, sampled tokens' h (bf16) and
    outputs against the oracle's W4A16 layer over the experts they use."""
    wl = W.WORKLOADS[name]
    dev = G.need_gpu()
    T, E, k = wl.T, wl.E, wl.k
    act = W.make_activations(wl, 0, dev)
    wts = W.make_weights(wl, 0, dev)
    experts = ops.NVFP4Experts.from_float(wts["w_gate"], wts["w_up"], wts["w_down"])
    x_bits = G.bf16_bits(act["x"])
    logits = act["logits"].cpu().numpy()
    ids_all, _ = O.route(logits, k)
    sample = checked_tokens(ids_all, T, E)
    perm = O.permute(ids_all, E)
    touched = np.unique(ids_all[sample])
    tt = torch.as_tensor(touched, device=dev)
    wg = G.quantize_experts_parallel(wts["w_gate"][tt].cpu().numpy())
    wu = G.quantize_experts_parallel(wts["w_up"][tt].cpu().numpy())
    wd = G.quantize_experts_parallel(wts["w_down"][tt].cpu().numpy())
    del wts
    ref = O.moe_ffn_w4a16(x_bits[sample], logits[sample][:, touched], k, wg, wu, wd)
    assert np.array_equal(touched[ref["ids"]], ids_all[sample])

    layer = ops.MoeFFN(experts, k, None, act=C.ACT_BF16)
    out = layer(act["x"], act["logits"])
    torch.cuda.synchronize()
    im = layer.intermediates(T)
    assert np.array_equal(im["topk_ids"].cpu().numpy(), ids_all)
    assert np.array_equal(im["counts"].cpu().numpy(), perm["counts"])
    assert np.array_equal(im["pair_to_row"].cpu().numpy(), perm["pair_to_row"])
    # sampled pairs' h rows, in the oracle's row order
    gpu_rows = perm["pair_to_row"][(sample[:, None] * k + np.arange(k)[None, :]).reshape(-1)]
    ref_rows = ref["pair_to_row"][np.arange(len(sample) * k)]
    hg = np.empty_like(ref["h_bf16"])
    hg[ref_rows] = im["h_bf16"].cpu().numpy().view(np.uint16)[gpu_rows]
    n_diff = G.check_h_bf16(hg, ref["h_bf16"])
    print(f"[full size w4a16] {name}: {len(sample)} tokens, {len(touched)} experts, {n_diff} h differ")
    G.check_out(G.bf16_bits(out)[sample], ref["out_f64"])


@pytest.mark.parametrize("name,launch", [("decode", "single"), ("dense_t1", "single"), ("decode", "single_local")])
def test_fullsize_calls_with_changing_routing(name, launch):
    """Consecutive calls whose routing differs (the workload's inputs, then all-zero inputs that
    send every token to the same experts, and so on): every call completes without a device
    timeout and every call on the workload's inputs gives the same output bit for bit.  The
    single-launch layer's stage ring is shared by two producers; this covers the case where one
    of them could otherwise run a full ring ahead of the stages being consumed."""
    wl = W.WORKLOADS[name]
    dev = G.need_gpu()
    act = W.make_activations(wl, 0, dev)
    wts = W.make_weights(wl, 0, dev)
    experts = ops.NVFP4Experts.from_float(wts["w_gate"], wts["w_up"], wts["w_down"])
    del wts
    mode = {"single": C.LAUNCH_SINGLE, "single_local": C.LAUNCH_SINGLE_LOCAL}[launch]
    layer = ops.MoeFFN(experts, wl.k, torch.full((wl.E,), 0.01, device=dev), launch=mode)
    assert layer.layout(wl.T).single_launch == 1
    ops.device_status(clear=True)
    first = layer(act["x"], act["logits"]).clone()
    zx, zl = torch.zeros_like(act["x"]), torch.zeros_like(act["logits"])
    for _ in range(4):
        layer(zx, zl)
        again = layer(act["x"], act["logits"])
        torch.cuda.synchronize()
        assert ops.device_status(clear=True) == 0
        assert torch.equal(again, first)
