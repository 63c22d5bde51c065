"""Shared helpers of the GPU parity tests: running the oracle and the library on the same
seeded inputs and applying the stated tolerances."""
from __future__ import annotations

import concurrent.futures as cf

import numpy as np
import torch

import oracle as O
from nvfp4_mixture_experts_w4a4_b200 import _lib as C
from nvfp4_mixture_experts_w4a4_b200 import ops, workloads as W
from tests.helpers import layouts as LY
from tests.helpers import refquant as R

# Output tolerance of the layer: |gpu - oracle| <= 1e-2 * max(|oracle|, RMS of the oracle row).
OUT_RTOL = 1e-2
# At most this fraction of requantised h codes may differ, each by one grid step.
H_CODE_FRAC = 1e-3


def need_gpu():
    if not torch.cuda.is_available():
        raise RuntimeError("this test needs a CUDA device")
    return torch.device("cuda:0")


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def quantize_experts_parallel(w: np.ndarray, nthreads: int | None = None):
    """Oracle quantisation of stacked weights [E, N, K] on several threads (ctypes releases
    the GIL while the oracle runs)."""
    E, N, K = w.shape
    codes = np.zeros((E, N, K // 2), np.uint8)
    sf = np.zeros((E, N, K // 16), np.uint8)
    sc = np.zeros(E, np.float32)

    def one(e):
        c, s, t = O.quantize(w[e])
        codes[e], sf[e], sc[e] = c, s, t

    with cf.ThreadPoolExecutor(nthreads or O.default_threads()) as ex:
        list(ex.map(one, range(E)))
    return codes, sf, sc


def check_out(gpu_bf16: np.ndarray, ref_f64: np.ndarray, rtol: float = OUT_RTOL, extra=None):
    """|gpu - oracle| <= rtol * max(|oracle|, row RMS) (+ `extra`, the propagated effect of
    the allowed one-grid-step differences of intermediate codes, when given)."""
    g = bits_to_f32(gpu_bf16).astype(np.float64)
    rms = np.sqrt((ref_f64 ** 2).mean(axis=1, keepdims=True))
    bound = rtol * np.maximum(np.abs(ref_f64), rms)
    if extra is not None:
        bound = bound + extra
    err = np.abs(g - ref_f64)
    ratio = err / np.maximum(bound, 1e-30)
    bad = err > bound
    if bad.any():
        t, n = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        raise AssertionError(
            f"{bad.sum()} of {bad.size} outputs outside tolerance; worst at [{t},{n}]: gpu={g[t, n]:.6g} "
            f"oracle={ref_f64[t, n]:.6g} err={err[t, n]:.3g} bound={bound[t, n]:.3g} row_rms={rms[t, 0]:.3g} "
            f"extra={0.0 if extra is None else extra[t, n]:.3g}")
    return float(ratio.max())


def _signed_index(codes: np.ndarray) -> np.ndarray:
    mag = (codes & 7).astype(np.int32)
    return np.where(codes & 8, -mag, mag)


def unpack(codes: np.ndarray) -> np.ndarray:
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 0xF
    out[..., 1::2] = codes >> 4
    return out


def check_h_codes(gpu_codes, gpu_sf, ref_codes, ref_sf, frac: float = H_CODE_FRAC):
    """Requantised h: at most `frac` of the codes differ; where the block scale agrees, a
    differing code is one grid step away (signed grid index within 1)."""
    gc, rc = unpack(gpu_codes), unpack(ref_codes)
    rows, K = gc.shape
    gs = np.repeat(gpu_sf, 16, axis=1)
    rs = np.repeat(ref_sf, 16, axis=1)
    same_sf = gs == rs
    differ = (gc != rc) | ~same_sf
    n = int(differ.sum())
    assert n <= frac * differ.size, f"{n} of {differ.size} h codes differ"
    step = np.abs(_signed_index(gc) - _signed_index(rc))
    # -0 and +0 are the same value
    zero_pair = ((gc & 7) == 0) & ((rc & 7) == 0)
    step = np.where(zero_pair, 0, step)
    assert (step[same_sf] <= 1).all(), "an h code differs by more than one grid step"
    return n


def layer_inputs(wl: W.Workload, seed: int = 0):
    """CPU-drawn inputs and oracle-quantised weights of a workload small enough to draw on the CPU."""
    act = W.make_activations(wl, seed, "cpu")
    wts = W.make_weights(wl, seed, "cpu")
    wg = quantize_experts_parallel(wts["w_gate"].numpy())
    wu = quantize_experts_parallel(wts["w_up"].numpy())
    wd = quantize_experts_parallel(wts["w_down"].numpy())
    return act, wts, wg, wu, wd


def experts_from_oracle(wg, wu, wd, dev) -> ops.NVFP4Experts:
    arrs = LY.experts_to_device_layout(wg, wu, wd)
    t = [torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in arrs]
    return ops.NVFP4Experts(*t)


def run_layer_pair(wl: W.Workload, path: int, seed: int = 0, dev=None, given_x_scale: bool = False,
                   combine: int = C.COMBINE_AUTO, dynamic_h: bool = False, launch: int = C.LAUNCH_AUTO):
    """Runs oracle and library on the same inputs; returns (oracle result, gpu out, layer).
    The oracle calibrates s_h (amax of each expert's h / 2688); the library is given those
    scales, or with dynamic_h derives its own in the call."""
    dev = dev or need_gpu()
    act, wts, wg, wu, wd = layer_inputs(wl, seed)
    x_bits = bf16_bits(act["x"])
    logits = act["logits"].numpy()
    xs = None
    if given_x_scale:
        xs = float(np.float32(np.abs(bits_to_f32(x_bits)).max()) / np.float32(2688) * np.float32(1.5))
    ref = O.moe_ffn(x_bits, logits, wl.k, wg, wu, wd, x_scale=xs)
    experts = experts_from_oracle(wg, wu, wd, dev)
    layer = ops.MoeFFN(experts, wl.k, None if dynamic_h else torch.from_numpy(ref["h_scale"]).to(dev),
                       x_scale=None if xs is None else torch.tensor([xs], device=dev), path=path, combine=combine,
                       launch=launch)
    h_amax = torch.empty(wl.E, dtype=torch.float32, device=dev)
    out = layer(act["x"].to(dev), act["logits"].to(dev), h_amax=h_amax)
    torch.cuda.synchronize()
    layer.oracle_wd = wd
    return ref, out, layer, h_amax


def check_layer(wl: W.Workload, ref: dict, out: torch.Tensor, layer: ops.MoeFFN, h_amax: torch.Tensor,
                wd=None):
    """wd: the oracle's (codes, sf, scale) of the down weights, used to bound the effect of
    differing h codes; when omitted, differing h codes get no output allowance."""
    wd = wd if wd is not None else getattr(layer, "oracle_wd", None)
    wd_dequant = None if wd is None else (lambda e: R.dequantize(wd[0][e], wd[1][e], wd[2][e]))
    T, k, H, I, E = wl.T, wl.k, wl.H, wl.I, wl.E
    im = layer.intermediates(T)
    # routing and permutation: bit-exact
    assert np.array_equal(im["topk_ids"].cpu().numpy(), ref["ids"])
    np.testing.assert_allclose(im["topk_w"].cpu().numpy(), ref["w"], rtol=2e-6, atol=1e-7)
    assert np.array_equal(im["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(im["offsets"].cpu().numpy(), ref["offsets"])
    # x scale and codes: bit-exact
    assert im["x_scale"].item() == np.float32(ref["x_scale"]) or layer.x_scale is not None
    p2r = im["pair_to_row"].cpu().numpy()
    if im["path"] == C.PATH_GEMV:
        assert np.array_equal(p2r, ref["pair_to_row"])
        assert np.array_equal(im["row_token"].cpu().numpy()[:T * k], ref["row_token"])
        xc = im["x_codes"].cpu().numpy()
        xsf = LY.from_mma(im["x_sf"].cpu().numpy(), T, H)
        assert np.array_equal(xc, ref["x_codes"])
        assert np.array_equal(xsf, ref["x_sf"])
        hrows = np.arange(T * k)
    else:
        po = im["padded_offsets"].cpu().numpy()
        off = ref["offsets"]
        counts = ref["counts"]
        mt = im["m_tile"]
        assert np.array_equal(po, np.concatenate([[0], np.cumsum((counts + mt - 1) // mt * mt)]))
        # padded row -> unpadded row: same expert, same rank
        e_of_pair = ref["ids"].reshape(-1)
        assert np.array_equal(p2r - po[e_of_pair] + off[e_of_pair], ref["pair_to_row"])
        hrows = p2r[np.argsort(ref["pair_to_row"])]  # padded row of each oracle row
        rt = im["row_token"].cpu().numpy()
        assert np.array_equal(rt[hrows], ref["row_token"])
        xc = im["x_codes"].cpu().numpy()[hrows]
        xsf = LY.from_mma(im["x_sf"].cpu().numpy(), im["x_rows"], H)[hrows]
        assert np.array_equal(xc, ref["x_codes"][ref["row_token"]])
        assert np.array_equal(xsf, ref["x_sf"][ref["row_token"]])
    # h: within the requantisation tolerance
    hc = im["h_codes"].cpu().numpy()[hrows]
    hsf = LY.from_mma(im["h_sf"].cpu().numpy(), im["h_rows"], I)[hrows]
    n_h_diff = check_h_codes(hc, hsf, ref["h_codes"], ref["h_sf"])
    # calibration output: amax of h per expert, within fp32 accumulation differences
    ha = h_amax.cpu().numpy()
    np.testing.assert_allclose(ha[ref["counts"] > 0], ref["h_amax"][ref["counts"] > 0], rtol=1e-4)
    # layer output: the oracle's output, with the bound widened by the first-order effect of
    # the (allowed, one-grid-step) h code differences on the rows where they occurred
    extra = None
    if n_h_diff and wd_dequant is not None:
        extra = h_diff_effect(hc, hsf, ref, wl, wd_dequant)
    print(f"[parity] {wl.name} T={T}: {n_h_diff} of {hc.size * 2} h codes differ")
    return check_out(bf16_bits(out), ref["out_f64"], extra=extra)


def h_diff_effect(hc, hsf, ref, wl, wd_dequant):
    """Per output element, sum over the differing h elements of w[t][j] * |dh| * |Wd[e][n][i]|,
    with dh the difference of the two dequantised values (both at the oracle's s_h)."""
    from tests.helpers import refquant as RQ
    T, H, k = wl.T, wl.H, wl.k
    s_h = ref["h_scale"]
    extra = np.zeros((T, H))
    gv = RQ.dequantize(hc, hsf, 1.0)
    rv = RQ.dequantize(ref["h_codes"], ref["h_sf"], 1.0)
    rows = np.nonzero((gv != rv).any(axis=1))[0]
    for r in rows:
        t, j = int(ref["row_token"][r]), int(ref["row_slot"][r])
        e = int(ref["ids"][t, j])
        dh = np.abs(gv[r] - rv[r]) * s_h[e]
        extra[t] += ref["w"][t, j] * (np.abs(wd_dequant(e)) @ dh)
    return extra


def run_layer_pair_w4a16(wl: W.Workload, seed: int = 0, dev=None, x_scale_log2=None):
    """The weight-only (W4A16) layer on the device and in the oracle, on the same inputs.
    x_scale_log2 (an int array shaped like x, or one value per token) multiplies x by those
    powers of two first (exact in bf16 while the results stay normal)."""
    dev = dev or need_gpu()
    act, wts, wg, wu, wd = layer_inputs(wl, seed)
    if x_scale_log2 is not None:
        e = np.asarray(x_scale_log2, np.float64)
        e = e.reshape(-1, 1) if e.ndim == 1 else e
        scaled = act["x"].double() * torch.from_numpy(np.exp2(e))
        act["x"] = scaled.to(torch.bfloat16)
        assert torch.equal(act["x"].double(), scaled), "the scaled x must be exact in bf16"
    ref = O.moe_ffn_w4a16(bf16_bits(act["x"]), act["logits"].numpy(), wl.k, wg, wu, wd)
    layer = ops.MoeFFN(experts_from_oracle(wg, wu, wd, dev), wl.k, None, act=C.ACT_BF16)
    out = layer(act["x"].to(dev), act["logits"].to(dev))
    torch.cuda.synchronize()
    return ref, out, layer


def check_h_bf16(gpu_bits: np.ndarray, ref_bits: np.ndarray, frac: float = H_CODE_FRAC) -> int:
    """Weight-only h (bf16 bit patterns, rows of one token-expert pair): equal except for at
    most `frac` of the elements, each one bf16 step away (a rounding boundary that the fp32
    sums of the device and the fp64 sums of the oracle put on different sides), or where g or
    u cancel: within 2^-16 of its row's largest |h| (the fp32 sums of the device carry an
    absolute error of that order there, the oracle's fp64 none).  Returns the differing count."""
    hg = gpu_bits.astype(np.int64)
    hr = ref_bits.astype(np.int64)
    diff = hg != hr
    assert diff.sum() <= frac * diff.size, f"{diff.sum()} of {diff.size} h values differ"
    vg = bits_to_f32(hg.astype(np.uint16)).astype(np.float64)
    vr = bits_to_f32(hr.astype(np.uint16)).astype(np.float64)
    # bit patterns of one sign are ordered like their values
    one_step = ((hg >> 15) == (hr >> 15)) & (np.abs(hg - hr) == 1)
    near_zero = np.abs(vg - vr) <= 2.0 ** -16 * np.abs(vr).max(axis=1, keepdims=True)
    bad = diff & ~one_step & ~near_zero
    assert not bad.any(), f"h differs beyond one bf16 step: gpu {vg[bad][:4]} oracle {vr[bad][:4]}"
    return int(diff.sum())


def check_layer_w4a16(wl: W.Workload, ref: dict, out: torch.Tensor, layer: ops.MoeFFN):
    """Routing and permutation bit-exact; h (bf16) equal except for at most H_CODE_FRAC of its
    elements, each one bf16 step away (a rounding boundary that the fp32 sums of the device
    and the fp64 sums of the oracle put on different sides); outputs within the tolerance."""
    T, k = wl.T, wl.k
    im = layer.intermediates(T)
    assert im["path"] == C.PATH_GEMV
    assert np.array_equal(im["topk_ids"].cpu().numpy(), ref["ids"])
    np.testing.assert_allclose(im["topk_w"].cpu().numpy(), ref["w"], rtol=2e-6, atol=1e-7)
    assert np.array_equal(im["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(im["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(im["pair_to_row"].cpu().numpy(), ref["pair_to_row"])
    n = check_h_bf16(im["h_bf16"].cpu().numpy().view(np.uint16), ref["h_bf16"])
    print(f"[parity w4a16] {wl.name} T={T}: {n} of {ref['h_bf16'].size} h values differ")
    return check_out(bf16_bits(out), ref["out_f64"])


def mx_experts(wts):
    """MXFP4 weights of a workload (oracle MX quantiser on the fp32 draws): dict of (codes, e8m0)
    per matrix, [E, N, K/2] and [E, N, K/32]."""
    out = {}
    for name in ("w_gate", "w_up", "w_down"):
        w = wts[name].numpy()
        mx = [O.mx_quantize(w[e]) for e in range(w.shape[0])]
        out[name] = (np.stack([m[0] for m in mx]), np.stack([m[1] for m in mx]))
    return out


def run_layer_pair_mxfp4(wl: W.Workload, path: int, act_mode: int = C.ACT_NVFP4, seed: int = 0, dev=None):
    """MXFP4 weights: the device converts them (NVFP4Experts.from_mxfp4), the oracle converts its
    own copy (reading R11); both layers then run on those weights."""
    dev = dev or need_gpu()
    act = W.make_activations(wl, seed, "cpu")
    wts = W.make_weights(wl, seed, "cpu")
    mx = mx_experts(wts)
    wg, wu, wd = (O.mx_experts_to_nvfp4(*mx[n]) for n in ("w_gate", "w_up", "w_down"))
    to = lambda t: torch.from_numpy(np.ascontiguousarray(t)).to(dev)  # noqa: E731
    experts = ops.NVFP4Experts.from_mxfp4(*((to(mx[n][0]), to(mx[n][1])) for n in ("w_gate", "w_up", "w_down")))
    torch.cuda.synchronize()
    ref_w = LY.experts_to_device_layout(wg, wu, wd)
    got_w = [experts.w13_codes, experts.w13_sf, experts.w13_scale, experts.w2_codes, experts.w2_sf, experts.w2_scale]
    for r, g in zip(ref_w, got_w):
        assert np.array_equal(g.cpu().numpy(), r)
    x_bits = bf16_bits(act["x"])
    logits = act["logits"].numpy()
    if act_mode == C.ACT_BF16:
        ref = O.moe_ffn_w4a16(x_bits, logits, wl.k, wg, wu, wd)
        layer = ops.MoeFFN(experts, wl.k, None, act=C.ACT_BF16)
    else:
        ref = O.moe_ffn(x_bits, logits, wl.k, wg, wu, wd)
        layer = ops.MoeFFN(experts, wl.k, torch.from_numpy(ref["h_scale"]).to(dev), path=path)
    h_amax = torch.empty(wl.E, dtype=torch.float32, device=dev)
    out = layer(act["x"].to(dev), act["logits"].to(dev), h_amax=None if act_mode == C.ACT_BF16 else h_amax)
    torch.cuda.synchronize()
    layer.oracle_wd = wd
    return ref, out, layer, h_amax


def shared_weights(wl: W.Workload, I_s: int, seed: int = 5):
    """A BF16 shared expert for a workload: gate/up [I_s, H] and down [H, I_s], N(0, 1/sqrt(fan_in))
    rounded to bf16; returned as bf16 bit patterns (oracle) and device tensors (library)."""
    g = torch.Generator().manual_seed(seed)
    gate = (torch.randn(I_s, wl.H, generator=g) / wl.H ** 0.5).to(torch.bfloat16)
    up = (torch.randn(I_s, wl.H, generator=g) / wl.H ** 0.5).to(torch.bfloat16)
    down = (torch.randn(wl.H, I_s, generator=g) / I_s ** 0.5).to(torch.bfloat16)
    bits = tuple(t.view(torch.int16).numpy().view(np.uint16) for t in (gate, up, down))
    return gate, up, down, bits


def run_layer_pair_shared(wl: W.Workload, path: int, I_s: int, act_mode: int = C.ACT_NVFP4,
                          combine: int = C.COMBINE_AUTO, seed: int = 0, dev=None):
    dev = dev or need_gpu()
    act, wts, wg, wu, wd = layer_inputs(wl, seed)
    gate, up, down, bits = shared_weights(wl, I_s)
    x_bits = bf16_bits(act["x"])
    logits = act["logits"].numpy()
    experts = experts_from_oracle(wg, wu, wd, dev)
    shared = (ops.shared_expert_w13(gate.to(dev), up.to(dev)), down.to(dev))
    if act_mode == C.ACT_BF16:
        ref = O.moe_ffn_w4a16(x_bits, logits, wl.k, wg, wu, wd, shared=bits)
        layer = ops.MoeFFN(experts, wl.k, None, act=C.ACT_BF16, shared=shared)
    else:
        ref = O.moe_ffn(x_bits, logits, wl.k, wg, wu, wd, shared=bits)
        layer = ops.MoeFFN(experts, wl.k, torch.from_numpy(ref["h_scale"]).to(dev), path=path, combine=combine,
                           shared=shared)
    h_amax = torch.empty(wl.E, dtype=torch.float32, device=dev)
    out = layer(act["x"].to(dev), act["logits"].to(dev), h_amax=None if act_mode == C.ACT_BF16 else h_amax)
    torch.cuda.synchronize()
    layer.oracle_wd = wd
    return ref, out, layer, h_amax
