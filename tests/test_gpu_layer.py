"""GPU parity of the whole routed layer (moe_ffn_forward through the C ABI) against the
CPU oracle: routing, permutation and activation codes bit-exact, requantised h within the
one-grid-step rule, outputs within 1e-2 * max(|oracle|, row RMS)."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_mixture_experts_w4a4_b200 import _lib as C
from nvfp4_mixture_experts_w4a4_b200 import ops, workloads as W
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

TINY = W.WORKLOADS["tiny"]
# reduced versions of the larger workloads that the oracle finishes in seconds, spanning
# several tiles and a ragged tail
CASES = {
    "tiny": TINY,
    "decode_small_E": W.scaled(W.WORKLOADS["decode"], E=64, H=1024, I=256),
    "decode_T1": W.scaled(W.WORKLOADS["decode"], T=1, E=64, H=1024, I=256),
    "prefill_chunk_small": W.scaled(W.WORKLOADS["prefill_chunk"], T=40, E=32, H=512, I=192),
    "long_prefill_small": W.scaled(W.WORKLOADS["long_prefill"], T=67, E=16, H=768, I=320, k=4),
    "dense_small": W.scaled(W.WORKLOADS["dense"], T=9, H=512, I=576),
    "top1_E2": W.scaled(TINY, T=13, E=2, k=1),
    "slices_E1024_k32": W.scaled(TINY, T=70, E=1024, k=32, H=256, I=128),
}


# the tensor-core path needs I % 128 == 0 (and H % 256 == 0)
GEMM_CASES = {
    "tiny": TINY,
    "prefill_chunk_small": W.scaled(W.WORKLOADS["prefill_chunk"], T=40, E=32, H=512, I=256),
    "long_prefill_small": W.scaled(W.WORKLOADS["long_prefill"], T=67, E=16, H=768, I=384, k=4),
    "dense_small": W.scaled(W.WORKLOADS["dense"], T=150, H=512, I=640),
    "one_expert_many_tiles": W.scaled(TINY, T=300, E=3, k=1, H=256, I=128),
    "decode_shape": W.scaled(W.WORKLOADS["decode"], E=64, H=1024, I=256),
    "decode_T1": W.scaled(W.WORKLOADS["decode"], T=1, E=64, H=1024, I=256),
    "popular_expert_chunks": W.scaled(W.WORKLOADS["prefill_chunk"], T=450, E=16, H=512, I=128, k=2),
    "slices_E1024_k32": W.scaled(TINY, T=97, E=1024, k=32, H=256, I=128),
}


@pytest.mark.parametrize("name", list(GEMM_CASES))
def test_layer_gemm_path(name):
    wl = GEMM_CASES[name]
    ref, out, layer, h_amax = G.run_layer_pair(wl, C.PATH_GEMM)
    assert layer.intermediates(wl.T)["path"] == C.PATH_GEMM
    G.check_layer(wl, ref, out, layer, h_amax)
    assert ops.device_status() == 0


@pytest.mark.parametrize("name", list(CASES))
def test_layer_gemv_path(name):
    wl = CASES[name]
    ref, out, layer, h_amax = G.run_layer_pair(wl, C.PATH_GEMV)
    G.check_layer(wl, ref, out, layer, h_amax)
    assert ops.device_status() == 0


def test_layer_given_x_scale():
    wl = CASES["decode_small_E"]
    ref, out, layer, h_amax = G.run_layer_pair(wl, C.PATH_GEMV, given_x_scale=True)
    G.check_layer(wl, ref, out, layer, h_amax)


def test_layer_all_tokens_one_expert_and_idle_experts():
    wl = W.scaled(TINY, T=21, E=6, k=2)
    dev = G.need_gpu()
    act, wts, wg, wu, wd = G.layer_inputs(wl, 3)
    logits = np.full((wl.T, wl.E), -4.0, np.float32)
    logits[:, 1] = 2.0           # every token's first choice
    logits[:, 5] = 0.5           # second choice of most tokens
    logits[::3, 4] = 1.0         # a third of the tokens take expert 4 second instead
    x_bits = G.bf16_bits(act["x"])
    ref = O.moe_ffn(x_bits, logits, wl.k, wg, wu, wd)
    assert ref["counts"][1] == wl.T and list(ref["counts"][[0, 2, 3]]) == [0, 0, 0]
    layer = ops.MoeFFN(G.experts_from_oracle(wg, wu, wd, dev), wl.k, torch.from_numpy(ref["h_scale"]).to(dev),
                       path=C.PATH_GEMV)
    h_amax = torch.empty(wl.E, device=dev)
    out = layer(act["x"].to(dev), torch.from_numpy(logits).to(dev), h_amax=h_amax)
    torch.cuda.synchronize()
    G.check_layer(wl, ref, out, layer, h_amax)


def test_layer_repeatable():
    wl = CASES["decode_small_E"]
    ref, out, layer, h_amax = G.run_layer_pair(wl, C.PATH_GEMV)
    act = W.make_activations(wl, 0, "cpu")
    again = layer(act["x"].cuda(), act["logits"].cuda())
    torch.cuda.synchronize()
    assert torch.equal(out, again)


def test_weights_quantised_on_gpu_match_oracle():
    """NVFP4Experts.from_float (the library quantiser, batched, gate/up interleaved) produces the
    oracle's codes, scales and tensor scales bit for bit."""
    wl = W.scaled(TINY, E=5, H=512, I=192)
    dev = G.need_gpu()
    wts = W.make_weights(wl, 0, "cpu")
    ex = ops.NVFP4Experts.from_float(wts["w_gate"].to(dev), wts["w_up"].to(dev), wts["w_down"].to(dev))
    torch.cuda.synchronize()
    wg = G.quantize_experts_parallel(wts["w_gate"].numpy())
    wu = G.quantize_experts_parallel(wts["w_up"].numpy())
    wd = G.quantize_experts_parallel(wts["w_down"].numpy())
    from tests.helpers import layouts as LY
    ref = LY.experts_to_device_layout(wg, wu, wd)
    got = [ex.w13_codes, ex.w13_sf, ex.w13_scale, ex.w2_codes, ex.w2_sf, ex.w2_scale]
    for r, g in zip(ref, got):
        assert np.array_equal(g.cpu().numpy(), r)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "prefill_chunk_small"])
def test_stage_marks_eager_and_in_a_cuda_graph(name):
    """Stage marks work on an eager call and inside a captured CUDA graph (where they are
    external event nodes), and neither the marks nor graph replay change the output."""
    wl = GEMM_CASES.get(name) or CASES[name]
    ref, out, layer, _ = G.run_layer_pair(wl, C.PATH_AUTO)
    dev = out.device
    act, *_ = G.layer_inputs(wl, 0)
    x, logits = act["x"].to(dev), act["logits"].to(dev)
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(C.STAGES)]
    eager = layer(x, logits, stage_events=marks)
    torch.cuda.synchronize()
    assert torch.equal(eager, out)
    times = [marks[i].elapsed_time(marks[i + 1]) for i in range(C.STAGES - 1)]
    assert all(t >= 0.0 for t in times) and sum(times) > 0.0

    graph_out = torch.empty_like(out)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        layer(x, logits, out=graph_out)
        side.synchronize()
        with torch.cuda.graph(g, stream=side):
            layer(x, logits, out=graph_out, stage_events=marks)
    torch.cuda.current_stream().wait_stream(side)
    graph_out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(graph_out, out)
    times = [marks[i].elapsed_time(marks[i + 1]) for i in range(C.STAGES - 1)]
    assert all(t >= 0.0 for t in times) and sum(times) > 0.0


@pytest.mark.parametrize("combine", [C.COMBINE_ORDERED, C.COMBINE_ACCUMULATE])
@pytest.mark.parametrize("name", ["tiny", "long_prefill_small", "dense_small", "popular_expert_chunks"])
def test_layer_gemm_combine_modes(name, combine):
    """Both ways of combining a token's k weighted rows (ordered fp32 slots; fp32 accumulation
    into the output rows) meet the stated tolerance, with either prologue."""
    wl = GEMM_CASES[name]
    ref, out, layer, h_amax = G.run_layer_pair(wl, C.PATH_GEMM, combine=combine)
    assert layer.intermediates(wl.T)["combine"] == combine
    G.check_layer(wl, ref, out, layer, h_amax)


def test_accumulate_needs_the_tensor_core_path():
    wl = CASES["long_prefill_small"]
    with pytest.raises(C.Nvfp4MoeError):
        G.run_layer_pair(wl, C.PATH_GEMV, combine=C.COMBINE_ACCUMULATE)


@pytest.mark.parametrize("name", ["tiny", "decode_shape", "decode_T1", "prefill_chunk_small", "long_prefill_small",
                                  "dense_small", "popular_expert_chunks", "slices_E1024_k32"])
def test_layer_dynamic_h_scale(name):
    """Dynamic per-expert h scale: the library derives s_h[e] = amax_e(h) / 2688 inside the
    call (h leaves the gate/up GEMM in fp32, then is requantised) and meets the same
    tolerances against the oracle's calibrating run; experts without tokens keep scale 1."""
    wl = GEMM_CASES[name]
    ref, out, layer, h_amax = G.run_layer_pair(wl, C.PATH_GEMM, dynamic_h=True)
    im = layer.intermediates(wl.T)
    used = ref["counts"] > 0
    s_dev = im["h_scale"].cpu().numpy()
    np.testing.assert_allclose(s_dev[used], ref["h_scale"][used], rtol=1e-4)
    assert (s_dev[~used] == 1.0).all()
    # the scale is the maximum divided by 2688, rounded once
    a_dev = im["h_amax"].cpu().numpy()
    assert np.array_equal(s_dev[used], a_dev[used] / np.float32(2688))
    assert np.array_equal(h_amax.cpu().numpy()[used], a_dev[used])
    G.check_layer(wl, ref, out, layer, h_amax)
    assert ops.device_status() == 0


@pytest.mark.parametrize("name", list(CASES))
def test_layer_weight_only_w4a16(name):
    """The weight-only variant (bf16 activations, NVFP4 weights, split-K GEMV) against the
    oracle's W4A16 layer."""
    wl = CASES[name]
    ref, out, layer = G.run_layer_pair_w4a16(wl)
    G.check_layer_w4a16(wl, ref, out, layer)
    assert ops.device_status() == 0


def test_weight_only_activations_outside_the_f16_range():
    """The weight-only products stage each token's bf16 activations in f16 times a power of two
    chosen from the token's largest magnitude.  Tokens scaled by 2^40, 2^24, 2^-24 and 2^-40
    (beyond f16's range either way), and tokens whose elements span 2^60 (half of them scaled by
    2^-60, far below f16's subnormals once the large half sets the power), must meet the same
    bounds as unscaled ones."""
    wl = CASES["decode_small_E"]
    per_token = np.array([40, 24, 0, -24, -40, 0, 12, -12] * ((wl.T + 7) // 8))[:wl.T]
    e = np.repeat(per_token[:, None], wl.H, axis=1)
    e[5::8, wl.H // 2:] = -60
    ref, out, layer = G.run_layer_pair_w4a16(wl, x_scale_log2=e)
    G.check_layer_w4a16(wl, ref, out, layer)
    assert ops.device_status() == 0


def test_weight_only_rejects_the_tensor_core_path():
    wl = CASES["tiny"]
    act, wts, wg, wu, wd = G.layer_inputs(wl)
    dev = G.need_gpu()
    layer = ops.MoeFFN(G.experts_from_oracle(wg, wu, wd, dev), wl.k, None, path=C.PATH_GEMM, act=C.ACT_BF16)
    with pytest.raises(C.Nvfp4MoeError):
        layer(act["x"].to(dev), act["logits"].to(dev))


@pytest.mark.parametrize("name,path,act", [("tiny", C.PATH_GEMM, C.ACT_NVFP4), ("decode_shape", C.PATH_GEMM, C.ACT_NVFP4),
                                           ("long_prefill_small", C.PATH_GEMM, C.ACT_NVFP4),
                                           ("tiny", C.PATH_GEMV, C.ACT_NVFP4), ("decode_shape", C.PATH_AUTO, C.ACT_BF16)])
def test_layer_mxfp4_weights(name, path, act):
    """MXFP4 weights on the NVFP4 layer: the device's exact NVFP4 form equals the oracle's
    (codes, scales, tensor scales, bit for bit), and the layer meets the usual tolerances."""
    wl = GEMM_CASES[name]
    ref, out, layer, h_amax = G.run_layer_pair_mxfp4(wl, path, act)
    if act == C.ACT_BF16:
        G.check_layer_w4a16(wl, ref, out, layer)
    else:
        G.check_layer(wl, ref, out, layer, h_amax)
    assert ops.device_status() == 0


@pytest.mark.parametrize("path,act", [(C.PATH_GEMM, C.ACT_NVFP4), (C.PATH_GEMV, C.ACT_NVFP4), (C.PATH_AUTO, C.ACT_BF16)])
def test_layer_empty_batch(path, act):
    """T = 0: the call succeeds, launches nothing and leaves an empty output."""
    wl = CASES["tiny"]
    dev = G.need_gpu()
    act_d, wts, wg, wu, wd = G.layer_inputs(wl)
    experts = G.experts_from_oracle(wg, wu, wd, dev)
    layer = ops.MoeFFN(experts, wl.k, None if act == C.ACT_BF16 else torch.ones(wl.E, device=dev), path=path, act=act)
    x = torch.empty(0, wl.H, dtype=torch.bfloat16, device=dev)
    logits = torch.empty(0, wl.E, dtype=torch.float32, device=dev)
    out = layer(x, logits)
    torch.cuda.synchronize()
    assert out.shape == (0, wl.H)
    assert ops.device_status() == 0


@pytest.mark.parametrize("name,path,act,combine", [
    ("tiny", C.PATH_GEMM, C.ACT_NVFP4, C.COMBINE_AUTO),
    ("decode_shape", C.PATH_GEMM, C.ACT_NVFP4, C.COMBINE_AUTO),
    ("long_prefill_small", C.PATH_GEMM, C.ACT_NVFP4, C.COMBINE_ORDERED),
    ("long_prefill_small", C.PATH_GEMM, C.ACT_NVFP4, C.COMBINE_ACCUMULATE),
    ("dense_small", C.PATH_GEMM, C.ACT_NVFP4, C.COMBINE_AUTO),
    ("tiny", C.PATH_GEMV, C.ACT_NVFP4, C.COMBINE_AUTO),
    ("decode_shape", C.PATH_AUTO, C.ACT_BF16, C.COMBINE_AUTO),
])
def test_layer_with_shared_expert(name, path, act, combine):
    """A BF16 shared expert beside the routed experts, added before the output's one rounding,
    on every path and combine mode, against the oracle (reading R12)."""
    wl = GEMM_CASES[name]
    ref, out, layer, h_amax = G.run_layer_pair_shared(wl, path, I_s=128 if wl.H <= 512 else 256, act_mode=act,
                                                      combine=combine)
    if act == C.ACT_BF16:
        G.check_layer_w4a16(wl, ref, out, layer)
    else:
        G.check_layer(wl, ref, out, layer, h_amax)
    assert ops.device_status() == 0


@pytest.mark.parametrize("name", ["tiny", "long_prefill_small"])
def test_graphed_layer_matches_eager(name):
    """The graph-replayed layer (ops.GraphedMoeFFN) gives the eager call's output bit for bit,
    from device and from pinned host inputs, call after call."""
    wl = GEMM_CASES[name]
    dev = G.need_gpu()
    act, wts, wg, wu, wd = G.layer_inputs(wl)
    experts = G.experts_from_oracle(wg, wu, wd, dev)
    layer = ops.MoeFFN(experts, wl.k, torch.ones(wl.E, device=dev) * 0.01)
    x, logits = act["x"].to(dev), act["logits"].to(dev)
    eager = layer(x, logits).clone()
    graphed = ops.GraphedMoeFFN(layer, wl.T)
    for src in ((x, logits), (act["x"].pin_memory(), act["logits"].pin_memory())):
        out = graphed(*src)
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    with pytest.raises(ValueError):
        graphed(x[:1], logits[:1])


@pytest.mark.parametrize("name", ["tiny", "decode_shape"])
def test_graphed_host_io_matches_eager(name):
    """With host_io the graph carries the transfers as well: x and logits from pinned host
    buffers, the output back to one.  Three different batches in turn (two passed to the call,
    one written into the host inputs in place) each give the eager call's output bit for bit."""
    wl = GEMM_CASES[name]
    dev = G.need_gpu()
    _, wts, wg, wu, wd = G.layer_inputs(wl)
    layer = ops.MoeFFN(G.experts_from_oracle(wg, wu, wd, dev), wl.k, torch.ones(wl.E, device=dev) * 0.01)
    graphed = ops.GraphedMoeFFN(layer, wl.T, host_io=True)
    for seed in (3, 4, 5):
        act = W.make_activations(wl, seed, "cpu")
        eager = layer(act["x"].to(dev), act["logits"].to(dev)).cpu()
        if seed == 5:
            graphed.x_host.copy_(act["x"])
            graphed.logits_host.copy_(act["logits"])
            out = graphed()
        else:
            out = graphed(act["x"], act["logits"])
        torch.cuda.current_stream().synchronize()
        assert not out.is_cuda
        assert torch.equal(out, eager)
    with pytest.raises(ValueError):
        graphed(act["x"].to(dev), act["logits"].to(dev))


# Batches of at most 16 tokens on the tensor-core path run the whole layer as one persistent
# launch (routing, permutation, x quantisation, both GEMMs, the ordered combine).
SINGLE_CASES = {
    "decode_E512_k10": W.scaled(W.WORKLOADS["decode"], E=512, H=1024, I=256),
    "k32_E1024": W.scaled(TINY, T=16, E=1024, k=32, H=256, I=256),
    "tiny_I128": TINY,
    "crowded_E4_T16": W.scaled(TINY, T=16, E=4, k=2, H=512, I=384),
    "ragged_T7": W.scaled(TINY, T=7, E=24, k=3, H=768, I=640),
    # K chunks of the down items: 2048 + 2048 + 512
    "dense_T1_three_chunks": W.scaled(W.WORKLOADS["dense"], T=1, H=512, I=4608),
    # a wide hidden size: fewer weight stages beside the resident x tile
    "dense_T3_H5120": W.scaled(W.WORKLOADS["dense"], T=3, H=5120, I=384),
}


@pytest.mark.parametrize("name", list(SINGLE_CASES))
def test_layer_single_launch(name):
    """The single-launch layer against the oracle with the usual tolerances, then called again
    on the same workspace: its counters and barrier start from zero in every call, so the second
    output is the first bit for bit."""
    wl = SINGLE_CASES[name]
    ref, out, layer, h_amax = G.run_layer_pair(wl, C.PATH_GEMM, launch=C.LAUNCH_SINGLE)
    assert layer.layout(wl.T).single_launch == 1
    G.check_layer(wl, ref, out, layer, h_amax)
    act = W.make_activations(wl, 0, "cpu")
    again = layer(act["x"].cuda(), act["logits"].cuda())
    torch.cuda.synchronize()
    assert torch.equal(out, again)
    assert ops.device_status() == 0


# Shapes with I % 256 == 0, run under both schedules of the single launch
SCHEDULE_CASES = {
    "decode_E512_k10": SINGLE_CASES["decode_E512_k10"],
    "k32_E1024": SINGLE_CASES["k32_E1024"],
    # 18 units of one expert: 18 CTAs with one unit each, the rest idle
    "dense_T1_18_units": SINGLE_CASES["dense_T1_three_chunks"],
    # four h chunks per expert and about 140 active experts: several units per CTA, so both
    # h buffers are reused and the down tiles of one unit follow the next unit's gate/up tiles
    "decode_I1024_units_per_cta": W.scaled(W.WORKLOADS["decode"], H=512, I=1024),
    "ragged_T5_I768": W.scaled(TINY, T=5, E=40, k=4, H=768, I=768),
}


@pytest.mark.parametrize("launch", ["tile", "local"])
@pytest.mark.parametrize("name", list(SCHEDULE_CASES))
def test_layer_single_launch_schedules(name, launch):
    """The single launch with its schedule forced (tile-level: h through global memory; expert-
    local: h chunks resident in shared memory) against the oracle, then called again: the
    second output is the first bit for bit."""
    wl = SCHEDULE_CASES[name]
    mode = {"tile": C.LAUNCH_SINGLE_TILE, "local": C.LAUNCH_SINGLE_LOCAL}[launch]
    ref, out, layer, h_amax = G.run_layer_pair(wl, C.PATH_GEMM, launch=mode)
    assert layer.layout(wl.T).single_launch == 1
    G.check_layer(wl, ref, out, layer, h_amax)
    act = W.make_activations(wl, 0, "cpu")
    again = layer(act["x"].cuda(), act["logits"].cuda())
    torch.cuda.synchronize()
    assert torch.equal(out, again)
    assert ops.device_status() == 0


def test_single_launch_selection():
    """LAUNCH_SINGLE takes the single launch where the batch allows it and is refused where it
    does not (17 tokens); the accumulating combine, a dynamic h scale or LAUNCH_MULTI keep the
    multi-launch path; LAUNCH_AUTO takes the single launch for the dense layer (one expert) and
    for routed decode batches that the expert-local schedule fits."""
    dev = G.need_gpu()
    wl = W.scaled(TINY, T=17)
    _, wts, wg, wu, wd = G.layer_inputs(wl)
    ex = G.experts_from_oracle(wg, wu, wd, dev)
    ones = torch.ones(wl.E, device=dev)
    single = lambda **kw: ops.MoeFFN(ex, wl.k, kw.pop("h", ones), launch=C.LAUNCH_SINGLE, **kw)  # noqa: E731
    assert single().layout(16).single_launch == 1
    assert single().layout(17).single_launch == 0
    with pytest.raises(C.Nvfp4MoeError):
        single()(torch.zeros(17, wl.H, dtype=torch.bfloat16, device=dev), torch.zeros(17, wl.E, device=dev))
    assert single(combine=C.COMBINE_ACCUMULATE).layout(16).single_launch == 0
    assert single(h=None).layout(16).single_launch == 0
    assert ops.MoeFFN(ex, wl.k, ones, launch=C.LAUNCH_MULTI).layout(16).single_launch == 0
    # the expert-local schedule needs I % 256 == 0 (here I = 128): refused, not rerouted
    local = ops.MoeFFN(ex, wl.k, ones, launch=C.LAUNCH_SINGLE_LOCAL)
    assert local.layout(16).single_launch == 0
    with pytest.raises(C.Nvfp4MoeError):
        local(torch.zeros(16, wl.H, dtype=torch.bfloat16, device=dev), torch.zeros(16, wl.E, device=dev))
    assert ops.MoeFFN(ex, wl.k, ones, launch=C.LAUNCH_SINGLE_TILE).layout(16).single_launch == 1
    dense = W.scaled(W.WORKLOADS["dense"], T=4, H=256, I=256)
    _, _, dg, du, dd = G.layer_inputs(dense)
    dex = G.experts_from_oracle(dg, du, dd, dev)
    assert ops.MoeFFN(dex, 1, torch.ones(1, device=dev)).layout(4).single_launch == 1
    # routed decode whose expected active experts fill the grid with expert-local units: AUTO
    # takes the single launch; at I = 128 (no local schedule) it keeps the multi-launch path
    E, H, I = 512, 256, 512
    gen = torch.Generator(device=dev).manual_seed(0)
    rex = ops.NVFP4Experts.from_float(torch.randn(E, I, H, device=dev, generator=gen),
                                      torch.randn(E, I, H, device=dev, generator=gen),
                                      torch.randn(E, H, I, device=dev, generator=gen))
    assert ops.MoeFFN(rex, 10, torch.ones(E, device=dev)).layout(16).single_launch == 1
    assert ops.MoeFFN(ex, wl.k, ones).layout(16).single_launch == 0
