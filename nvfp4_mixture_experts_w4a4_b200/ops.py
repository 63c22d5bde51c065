"""PyTorch-facing binding of libnvfp4moe: the C ABI's entry points under the same names.

Every function here only marshals arguments: it allocates outputs and workspaces with torch
(device memory is torch's job), passes raw device pointers and the current CUDA stream to
the library, and raises on a non-OK status.  All arithmetic runs in the library's kernels.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib as C
from ._lib import check, lib

__all__ = [
    "nvfp4_quantize", "moe_route", "moe_permute", "nvfp4_gemm", "moe_ffn_forward", "codec_convert",
    "device_status", "sf_mma_bytes", "NVFP4Experts", "MoeFFN",
]


def _p(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream=None):
    st = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(st.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libnvfp4moe takes CUDA tensors only")


def sf_mma_bytes(rows: int, K: int) -> int:
    return ((rows + 127) // 128) * 128 * (K // 16)


def _sf_bytes(rows: int, K: int, layout: int) -> int:
    return sf_mma_bytes(rows, K) if layout == C.SF_MMA else rows * (K // 16)


def codec_convert(x: torch.Tensor):
    """fp32 -> (E2M1 code per byte, E4M3 byte) with the kernels' element encoders."""
    _need_cuda(x)
    x = x.contiguous().view(-1)
    e2m1 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    e4m3 = torch.empty_like(e2m1)
    check(lib().nvfp4_codec_convert(_p(x), x.numel(), _p(e2m1), _p(e4m3), _s()), "nvfp4_codec_convert")
    return e2m1, e4m3


def device_status(clear: bool = True) -> int:
    v = ctypes.c_uint32(0)
    check(lib().nvfp4moe_device_status(_s(), int(clear), ctypes.byref(v)), "nvfp4moe_device_status")
    return int(v.value)


def mma_peak_tflops(iters: int = 20000, repeats: int = 3) -> float:
    """Measured block-scaled FP4 tensor-core ceiling of the current device in TFLOP/s: the
    best of `repeats` timed launches of nvfp4moe_mma_peak_probe (after one warm-up launch),
    CUDA events on the current stream."""
    s = torch.cuda.current_stream()
    check(lib().nvfp4moe_mma_peak_probe(max(1, iters // 10), _s()), "nvfp4moe_mma_peak_probe")
    best = float("inf")
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        check(lib().nvfp4moe_mma_peak_probe(iters, _s()), "nvfp4moe_mma_peak_probe")
        b.record(s)
        b.synchronize()
        best = min(best, a.elapsed_time(b))
    return lib().nvfp4moe_mma_peak_probe_flops(iters) / (best * 1e-3) / 1e12


def wait_selftest(polls: int) -> int:
    """Runs the bounded-wait self-test kernel (a wait on a barrier nothing arrives on, limited
    to `polls` polls) and returns its result word: 0 when the wait gave up."""
    r = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    check(lib().nvfp4moe_wait_selftest(polls, _p(r), _s()), "nvfp4moe_wait_selftest")
    return int(r.item())


def nvfp4_quantize(x: torch.Tensor, tensor_scale: torch.Tensor | None = None, *, sf_layout: int = C.SF_MMA,
                   row_gather: torch.Tensor | None = None, out_rows: int | None = None,
                   codes: torch.Tensor | None = None, sf: torch.Tensor | None = None,
                   scale_out: torch.Tensor | None = None):
    """Quantises x ([rows, K] or [batch, rows, K], bf16 or fp32) to NVFP4.

    tensor_scale: None -> dynamic (amax / 2688 per batch item, returned); otherwise a CUDA
    fp32 tensor with one scale per batch item.  Returns (codes, sf, scale) where codes is
    uint8 [batch?, out_rows, K/2] and sf uint8 [batch?, sf bytes] in `sf_layout`.
    """
    _need_cuda(x, tensor_scale, row_gather)
    squeeze = x.dim() == 2
    x3 = x.unsqueeze(0) if squeeze else x
    if x3.stride(-1) != 1:
        raise ValueError("x must have unit stride along K")
    B, rows, K = x3.shape
    if x3.dtype == torch.bfloat16:
        dt = C.DTYPE_BF16
    elif x3.dtype == torch.float32:
        dt = C.DTYPE_F32
    else:
        raise ValueError("x must be bf16 or fp32")
    orow = rows if row_gather is None else int(out_rows if out_rows is not None else row_gather.numel())
    dev = x.device
    if codes is None:
        codes = torch.empty(B, orow, K // 2, dtype=torch.uint8, device=dev)
    sfb = _sf_bytes(orow, K, sf_layout)
    if sf is None:
        sf = torch.empty(B, sfb, dtype=torch.uint8, device=dev)
    dynamic = tensor_scale is None
    if dynamic:
        scale = scale_out if scale_out is not None else torch.empty(B, dtype=torch.float32, device=dev)
    else:
        scale = tensor_scale.to(torch.float32).contiguous().view(-1)
    wsb = lib().nvfp4_quantize_workspace_size(B, rows, K) if dynamic else 0
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    rg = None if row_gather is None else row_gather.to(torch.int32).contiguous()
    st = lib().nvfp4_quantize(
        _p(x3), dt, B, rows, K, x3.stride(1), x3.stride(0) if B > 1 else rows * x3.stride(1), _p(rg), orow,
        C.SCALE_DYNAMIC if dynamic else C.SCALE_GIVEN, _p(scale), _p(codes),
        codes.stride(0) if codes.dim() == 3 else 0, _p(sf), sf.stride(0) if sf.dim() == 2 else 0,
        sf_layout, _p(ws), wsb, _s())
    check(st, "nvfp4_quantize")
    if squeeze:
        return codes[0], sf[0], scale
    return codes, sf, scale


def moe_route(logits: torch.Tensor, k: int):
    """Top-k expert ids (int32 [T, k]) and softmax-over-k weights (fp32 [T, k])."""
    _need_cuda(logits)
    logits = logits.to(torch.float32).contiguous()
    T, E = logits.shape
    ids = torch.empty(T, k, dtype=torch.int32, device=logits.device)
    w = torch.empty(T, k, dtype=torch.float32, device=logits.device)
    check(lib().moe_route(_p(logits), T, E, k, _p(ids), _p(w), _s()), "moe_route")
    return ids, w


def moe_permute(ids: torch.Tensor, E: int, m_tile: int = 1, zero_f32: torch.Tensor | None = None) -> dict:
    _need_cuda(ids)
    ids = ids.to(torch.int32).contiguous()
    T, k = ids.shape
    cap = int(lib().moe_permute_rows_capacity(T, E, k, m_tile))
    dev = ids.device
    i32 = dict(dtype=torch.int32, device=dev)
    r = dict(
        counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
        padded_offsets=torch.empty(E + 1, **i32), pair_to_row=torch.empty(max(T * k, 1), **i32),
        row_token=torch.empty(max(cap, 1), **i32), row_pair=torch.empty(max(cap, 1), **i32),
        tile_expert=torch.empty(max(cap // m_tile, 1), **i32), active=torch.empty(E + 1, **i32),
    )
    st = lib().moe_permute(_p(ids), T, E, k, m_tile, cap, _p(r["counts"]), _p(r["offsets"]),
                           _p(r["padded_offsets"]), _p(r["pair_to_row"]), _p(r["row_token"]),
                           _p(r["row_pair"]), _p(r["tile_expert"]), _p(r["active"]), _p(zero_f32), _s())
    check(st, "moe_permute")
    r["rows_cap"] = cap
    return r


def nvfp4_gemm(A: torch.Tensor, A_sf: torch.Tensor, a_scale: torch.Tensor, B: torch.Tensor, B_sf: torch.Tensor,
               b_scale: torch.Tensor, out_dtype=torch.bfloat16) -> torch.Tensor:
    """D = (A . B^T) * a_scale * b_scale for NVFP4 A [M, K/2] and B [N, K/2] (MMA-layout scales)."""
    _need_cuda(A, A_sf, a_scale, B, B_sf, b_scale)
    M, N, K = A.shape[0], B.shape[0], A.shape[1] * 2
    D = torch.empty(M, N, dtype=out_dtype, device=A.device)
    wsb = lib().nvfp4_gemm_workspace_size(M, N, K)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=A.device)
    dt = C.DTYPE_F32 if out_dtype == torch.float32 else C.DTYPE_BF16
    st = lib().nvfp4_gemm(_p(A), _p(A_sf), _p(a_scale), _p(B), _p(B_sf), _p(b_scale), M, N, K, _p(D), dt,
                          _p(ws), wsb, _s())
    check(st, "nvfp4_gemm")
    return D


def nvfp4_from_mxfp4(codes: torch.Tensor, e8m0: torch.Tensor, row_gather: torch.Tensor | None = None,
                     out_rows: int | None = None, codes_out: torch.Tensor | None = None,
                     sf_out: torch.Tensor | None = None):
    """The exact NVFP4 form of MXFP4 matrices codes [B, rows, K/2] / [rows, K/2] with E8M0 scales
    [.., rows, K/32]: returns (codes, MMA-layout sf [B, sf_mma_bytes(out_rows, K)], tensor scale [B]).
    Synchronous; raises when a matrix has no exact form."""
    _need_cuda(codes, e8m0)
    squeeze = codes.dim() == 2
    if squeeze:
        codes, e8m0 = codes[None], e8m0[None]
    codes, e8m0 = codes.contiguous(), e8m0.contiguous()
    B, rows, K = codes.shape[0], codes.shape[1], codes.shape[2] * 2
    out_rows = rows if out_rows is None else out_rows
    dev = codes.device
    if sf_out is None:
        sf_out = torch.empty(B, sf_mma_bytes(out_rows, K), dtype=torch.uint8, device=dev)
    scale = torch.empty(B, dtype=torch.float32, device=dev)
    wsb = lib().nvfp4_from_mxfp4_workspace_size(B)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    gather = None if row_gather is None else row_gather.to(torch.int32).contiguous()
    st = lib().nvfp4_from_mxfp4(_p(codes), _p(e8m0), B, rows, K, _p(gather), out_rows, _p(codes_out), _p(sf_out),
                                _p(scale), _p(ws), wsb, _s())
    check(st, "nvfp4_from_mxfp4")
    out_codes = codes if codes_out is None else codes_out
    if squeeze:
        return out_codes[0], sf_out[0], scale
    return out_codes, sf_out, scale


def nvfp4_prep_weights(codes: torch.Tensor | None, sf: torch.Tensor, K: int, *, rows: int | None = None,
                       sf_layout: int = C.SF_ROWMAJOR, row_gather: torch.Tensor | None = None,
                       out_rows: int | None = None, codes_out: torch.Tensor | None = None,
                       sf_out: torch.Tensor | None = None, sf_out_layout: int = C.SF_MMA):
    """Already-quantised NVFP4 matrices into the layer's layout (bytes only): out row r takes
    input row row_gather[r] (None: r; negative: left untouched), its codes copied to codes_out
    and its block scales written in sf_out_layout.  codes [B, rows, K/2] or [rows, K/2], or None
    to convert the scales alone (then give `rows`); sf [B, n] or [n] in sf_layout.  Returns
    (codes_out or None, sf_out).  A gather entry >= rows is skipped and reported in the device
    status word (DEV_BAD_GATHER)."""
    _need_cuda(sf, codes, row_gather)
    single = codes.dim() == 2 if codes is not None else sf.dim() == 1
    if codes is not None:
        codes = (codes[None] if single else codes).contiguous()
        rows = codes.shape[1]
    elif rows is None:
        raise ValueError("rows is required when only the scales are converted")
    sf = (sf.reshape(1, -1) if single else sf.reshape(sf.shape[0], -1)).contiguous()
    B = sf.shape[0]
    out_rows = rows if out_rows is None else out_rows
    dev = sf.device
    # outputs the call allocates are [B, ...] and lose the batch axis again for a single matrix;
    # the caller's own come back as they were given
    ret_codes, ret_sf = codes_out, sf_out
    if codes is not None and codes_out is None:
        codes_out = torch.empty(B, out_rows, K // 2, dtype=torch.uint8, device=dev)
        ret_codes = codes_out[0] if single else codes_out
    if sf_out is None:
        n = sf_mma_bytes(out_rows, K) if sf_out_layout == C.SF_MMA else out_rows * (K // 16)
        sf_out = torch.empty(B, n, dtype=torch.uint8, device=dev)
        ret_sf = sf_out[0] if single else sf_out
    def per_matrix(layout, n_rows):
        return sf_mma_bytes(n_rows, K) if layout == C.SF_MMA else n_rows * (K // 16)

    if sf.shape[1] != per_matrix(sf_layout, rows):
        raise ValueError(f"sf holds {sf.shape[1]} bytes per matrix, {per_matrix(sf_layout, rows)} expected")
    if sf_out.numel() != B * per_matrix(sf_out_layout, out_rows) or not sf_out.is_contiguous():
        raise ValueError("sf_out must be contiguous, one matrix of scales per batch item")
    if codes_out is not None and (codes_out.numel() != B * out_rows * (K // 2) or not codes_out.is_contiguous()):
        raise ValueError("codes_out must be contiguous [B, out_rows, K/2]")
    gather = None if row_gather is None else row_gather.to(torch.int32).contiguous()
    st = lib().nvfp4_prep_weights(_p(codes), _p(sf), sf_layout, B, rows, K, _p(gather), out_rows,
                                  _p(codes_out), _p(sf_out), sf_out_layout, _s())
    check(st, "nvfp4_prep_weights")
    return ret_codes, ret_sf


def shared_expert_w13(gate: torch.Tensor, up: torch.Tensor) -> torch.Tensor:
    """bf16 gate and up [I_s, H] of a shared expert -> the interleaved [2 I_s, H] the layer takes
    (rows 32c+j: gate row 16c+j for j < 16, up row 16c+j-16 otherwise); a setup-time layout step."""
    I, H = gate.shape
    if I % 16 or up.shape != gate.shape:
        raise ValueError("gate and up must both be [I_s, H] with I_s a multiple of 16")
    out = torch.empty(2 * I, H, dtype=gate.dtype, device=gate.device)
    groups = out.view(I // 16, 2, 16, H)  # row 32c+j = groups[c, j // 16, j % 16]
    groups[:, 0].copy_(gate.reshape(I // 16, 16, H))
    groups[:, 1].copy_(up.reshape(I // 16, 16, H))
    return out


class NVFP4Experts:
    """Per-expert NVFP4 weights in the library's layout (W13 interleaved, MMA scales)."""

    def __init__(self, w13_codes, w13_sf, w13_scale, w2_codes, w2_sf, w2_scale):
        self.w13_codes, self.w13_sf, self.w13_scale = w13_codes, w13_sf, w13_scale
        self.w2_codes, self.w2_sf, self.w2_scale = w2_codes, w2_sf, w2_scale
        self.E, twoI, h2 = w13_codes.shape
        self.I, self.H = twoI // 2, h2 * 2

    @staticmethod
    def interleave_maps(I: int, device) -> tuple[torch.Tensor, torch.Tensor]:
        """Row gathers that place gate rows at W13 rows 32c+j (j<16) and up rows at 32c+16+j
        (-1: the row is the other matrix's).  Built on the host and copied to the device once;
        the library's gathers (nvfp4_quantize, nvfp4_prep_weights, nvfp4_from_mxfp4) apply them."""
        r = np.arange(2 * I, dtype=np.int32)
        c, j = r // 32, r % 32
        gate = np.where(j < 16, 16 * c + j, -1).astype(np.int32)
        up = np.where(j >= 16, 16 * c + j - 16, -1).astype(np.int32)
        return torch.from_numpy(gate).to(device), torch.from_numpy(up).to(device)

    @classmethod
    def from_mxfp4(cls, gate: tuple, up: tuple, down: tuple) -> "NVFP4Experts":
        """MXFP4 expert weights, each (codes [E, N, K/2], E8M0 scales [E, N, K/32]) for gate/up
        [E, I, H] and down [E, H, I], in their exact NVFP4 form (nvfp4_from_mxfp4)."""
        E, I, h2 = gate[0].shape
        H = h2 * 2
        dev = gate[0].device
        g_map, u_map = cls.interleave_maps(I, dev)
        w13_codes = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=dev)
        w13_sf = torch.empty(E, sf_mma_bytes(2 * I, H), dtype=torch.uint8, device=dev)
        _, _, sg = nvfp4_from_mxfp4(gate[0], gate[1], g_map, 2 * I, w13_codes, w13_sf)
        _, _, su = nvfp4_from_mxfp4(up[0], up[1], u_map, 2 * I, w13_codes, w13_sf)
        w2_codes, w2_sf, sd = nvfp4_from_mxfp4(down[0], down[1])
        return cls(w13_codes, w13_sf, torch.stack([sg, su], 1).contiguous(), w2_codes.contiguous(), w2_sf,
                   sd.contiguous())

    @classmethod
    def from_nvfp4(cls, gate: tuple, up: tuple, down: tuple, sf_layout: int = C.SF_ROWMAJOR) -> "NVFP4Experts":
        """Expert weights already quantised to NVFP4, each (codes [E, N, K/2], block scales in
        sf_layout [E, ...], tensor scales [E]) for gate/up [E, I, H] and down [E, H, I]:
        gate and up interleaved into W13 and every block scale moved to the MMA layout
        (nvfp4_prep_weights); the tensor scales are kept as they are."""
        E, I, h2 = gate[0].shape
        H = h2 * 2
        dev = gate[0].device
        g_map, u_map = cls.interleave_maps(I, dev)
        w13_codes = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=dev)
        w13_sf = torch.empty(E, sf_mma_bytes(2 * I, H), dtype=torch.uint8, device=dev)
        nvfp4_prep_weights(gate[0], gate[1], H, sf_layout=sf_layout, row_gather=g_map, out_rows=2 * I,
                           codes_out=w13_codes, sf_out=w13_sf)
        nvfp4_prep_weights(up[0], up[1], H, sf_layout=sf_layout, row_gather=u_map, out_rows=2 * I,
                           codes_out=w13_codes, sf_out=w13_sf)
        w2_codes, w2_sf = nvfp4_prep_weights(down[0], down[1], I, sf_layout=sf_layout)
        w13_scale = torch.stack([gate[2].float(), up[2].float()], 1).contiguous()
        return cls(w13_codes, w13_sf, w13_scale, w2_codes, w2_sf, down[2].float().contiguous())

    @classmethod
    def from_float(cls, w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor) -> "NVFP4Experts":
        """Quantises fp32 weights [E, I, H] / [E, H, I] with one dynamic scale per expert and matrix."""
        E, I, H = w_gate.shape
        dev = w_gate.device
        g_map, u_map = cls.interleave_maps(I, dev)
        w13_codes = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=dev)
        w13_sf = torch.empty(E, sf_mma_bytes(2 * I, H), dtype=torch.uint8, device=dev)
        _, _, sg = nvfp4_quantize(w_gate, None, row_gather=g_map, out_rows=2 * I, codes=w13_codes, sf=w13_sf)
        _, _, su = nvfp4_quantize(w_up, None, row_gather=u_map, out_rows=2 * I, codes=w13_codes, sf=w13_sf)
        w2_codes, w2_sf, sd = nvfp4_quantize(w_down, None)
        return cls(w13_codes, w13_sf, torch.stack([sg, su], 1).contiguous(), w2_codes, w2_sf, sd.contiguous())


class MoeFFN:
    """The routed NVFP4 W4A4 feed-forward layer (moe_ffn_forward) with a cached workspace."""

    def __init__(self, experts: NVFP4Experts, top_k: int, h_scale: torch.Tensor | None,
                 x_scale: torch.Tensor | None = None, path: int = C.PATH_AUTO, combine: int = C.COMBINE_AUTO,
                 act: int = C.ACT_NVFP4, shared: tuple | None = None, launch: int = C.LAUNCH_AUTO):
        """h_scale: per-expert requantisation scales of h, or None for the dynamic scale
        (amax of each expert's h in the call / 2688; tensor-core path).  act: ACT_NVFP4 (W4A4)
        or ACT_BF16 (weight-only W4A16: bf16 activations, the GEMV path; no scales used).
        shared: None or a BF16 shared expert (w13 bf16 [2I_s, H] interleaved, see
        shared_expert_w13; w2 bf16 [H, I_s]), added to every token's output.  launch: LAUNCH_AUTO,
        LAUNCH_SINGLE (the whole layer as one persistent launch, where the batch allows it; the
        schedule, expert-local or tile-level, is chosen per call from the routing),
        LAUNCH_SINGLE_TILE / LAUNCH_SINGLE_LOCAL (the single launch with that schedule) or
        LAUNCH_MULTI (prologue, grouped GEMMs, combine)."""
        self.w = experts
        self.top_k = top_k
        self.h_scale = None if h_scale is None else h_scale.to(torch.float32).contiguous()
        self.x_scale = None if x_scale is None else x_scale.to(torch.float32).contiguous().view(1)
        self.path = path
        self.combine = combine
        self.act = act
        self.shared = None if shared is None else tuple(t.contiguous() for t in shared)
        self.launch = launch
        self._ws = {}    # size class (bytes) -> buffer
        self._need = {}  # T -> workspace bytes

    def desc(self, T: int, h_amax: torch.Tensor | None = None, events=None) -> C.MoeFfnDesc:
        w = self.w
        d = C.MoeFfnDesc()
        d.T, d.H, d.I, d.E, d.top_k = T, w.H, w.I, w.E, self.top_k
        d.path = self.path
        d.combine = self.combine
        d.x_scale_mode = C.SCALE_DYNAMIC if self.x_scale is None else C.SCALE_GIVEN
        d.x_scale = None if self.x_scale is None else self.x_scale.data_ptr()
        d.w13_codes, d.w13_sf, d.w13_scale = w.w13_codes.data_ptr(), w.w13_sf.data_ptr(), w.w13_scale.data_ptr()
        d.w2_codes, d.w2_sf, d.w2_scale = w.w2_codes.data_ptr(), w.w2_sf.data_ptr(), w.w2_scale.data_ptr()
        d.h_scale = None if self.h_scale is None else self.h_scale.data_ptr()
        d.h_scale_mode = C.SCALE_DYNAMIC if self.h_scale is None else C.SCALE_GIVEN
        d.h_amax = None if h_amax is None else h_amax.data_ptr()
        d.act_mode = self.act
        d.launch_mode = self.launch
        if self.shared is not None:
            d.shared_I = self.shared[1].shape[1]
            d.shared_w13, d.shared_w2 = self.shared[0].data_ptr(), self.shared[1].data_ptr()
        d.stage_events = None if events is None else ctypes.cast(events, ctypes.c_void_p).value
        return d

    def layout(self, T: int) -> C.MoeFfnWsLayout:
        L = C.MoeFfnWsLayout()
        d = self.desc(T)
        check(lib().moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L)), "moe_ffn_workspace_layout")
        return L

    def workspace(self, T: int) -> torch.Tensor:
        """The device workspace of a T-token call.  Workspaces are pooled by power-of-two size
        class (at least 1 MiB): batch sizes whose needs fall in one class share a buffer, so
        serving many batch sizes costs at most twice the largest need in total rather than one
        buffer per size.  A buffer is never freed, so a CUDA graph that captured a call keeps a
        valid workspace; calls on one layer must be ordered (one stream), as each call uses the
        whole workspace."""
        if T not in self._need:
            self._need[T] = max(int(self.layout(T).total), 16)
        need = self._need[T]
        size_class = max(1 << 20, 1 << (need - 1).bit_length())
        if size_class not in self._ws:
            self._ws[size_class] = torch.empty(size_class, dtype=torch.uint8, device=self.w.w13_codes.device)
        return self._ws[size_class]

    def forward(self, x: torch.Tensor, logits: torch.Tensor, out: torch.Tensor | None = None,
                h_amax: torch.Tensor | None = None, stage_events=None) -> torch.Tensor:
        """stage_events: optional list of 7 torch.cuda.Event (enable_timing) recorded at the
        layer's stage boundaries (see NVFP4MOE_STAGES)."""
        _need_cuda(x, logits, out, h_amax)
        w = self.w
        if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != w.H:
            raise ValueError(f"x must be bf16 [T, {w.H}], got {x.dtype} {tuple(x.shape)}")
        T = x.shape[0]
        if tuple(logits.shape) != (T, w.E):
            raise ValueError(f"logits must be [{T}, {w.E}], got {tuple(logits.shape)}")
        if out is not None and (out.dtype != torch.bfloat16 or tuple(out.shape) != (T, w.H)
                                or not out.is_contiguous()):
            raise ValueError(f"out must be a contiguous bf16 [{T}, {w.H}] tensor")
        if h_amax is not None and (h_amax.dtype != torch.float32 or h_amax.numel() != w.E
                                   or not h_amax.is_contiguous()):
            raise ValueError(f"h_amax must be a contiguous fp32 tensor of {w.E} values")
        x = x.contiguous()
        logits = logits.to(torch.float32).contiguous()
        if out is None:
            out = torch.empty(T, self.w.H, dtype=torch.bfloat16, device=x.device)
        ws = self.workspace(T)
        ev = None
        if stage_events is not None:
            if len(stage_events) != C.STAGES:
                raise ValueError(f"stage_events needs {C.STAGES} events")
            for e in stage_events:
                if not e.cuda_event:  # torch creates the event lazily: materialise it
                    e.record()
            ev = (ctypes.c_void_p * C.STAGES)(*[e.cuda_event for e in stage_events])
        d = self.desc(T, h_amax, ev)
        st = lib().moe_ffn_forward(ctypes.byref(d), _p(x), _p(logits), _p(out), _p(ws), ws.numel(), _s())
        check(st, "moe_ffn_forward")
        return out

    __call__ = forward

    def intermediates(self, T: int) -> dict:
        """Views of the intermediates of the last forward with T tokens (for inspection)."""
        L = self.layout(T)
        ws = self.workspace(T)
        w, k = self.w, self.top_k
        P = T * k

        def view(off, n, dtype):
            nbytes = n * torch.tensor([], dtype=dtype).element_size()
            return ws[off:off + nbytes].view(dtype)

        dyn_h = self.h_scale is None
        return dict(
            path=L.path, m_tile=L.m_tile, combine=L.combine,
            # the scales h was requantised with: given, or derived in the call (amax / 2688)
            h_scale=view(L.h_stats + 4 * w.E, w.E, torch.float32) if dyn_h else self.h_scale,
            h_amax=view(L.h_stats, w.E, torch.float32) if dyn_h else None,
            topk_ids=view(L.topk_ids, P, torch.int32).view(T, k),
            topk_w=view(L.topk_w, P, torch.float32).view(T, k),
            counts=view(L.counts, w.E, torch.int32), offsets=view(L.offsets, w.E + 1, torch.int32),
            padded_offsets=view(L.padded_offsets, w.E + 1, torch.int32),
            pair_to_row=view(L.pair_to_row, P, torch.int32),
            row_token=view(L.row_token, L.h_rows if L.path == C.PATH_GEMM else P, torch.int32),
            row_pair=view(L.row_pair, L.h_rows if L.path == C.PATH_GEMM else P, torch.int32),
            active=view(L.active, w.E + 1, torch.int32),
            x_scale=view(L.x_scale, 1, torch.float32),
            x_codes=view(L.x_codes, L.x_rows * w.H // 2, torch.uint8).view(L.x_rows, w.H // 2),
            x_sf=view(L.x_sf, sf_mma_bytes(L.x_rows, w.H), torch.uint8),
            h_codes=view(L.h_codes, L.h_rows * w.I // 2, torch.uint8).view(L.h_rows, w.I // 2),
            h_sf=view(L.h_sf, sf_mma_bytes(L.h_rows, w.I), torch.uint8),
            x_rows=L.x_rows, h_rows=L.h_rows,
            h_bf16=view(L.h_bf16, P * w.I, torch.int16).view(P, w.I) if self.act == C.ACT_BF16 else None,
        )


class GraphedMoeFFN:
    """The layer for a fixed batch size T, captured once into a CUDA graph over static buffers:
    a call copies x and logits into the static inputs (device or pinned host tensors), replays
    the graph (the same kernels as an eager call, without the per-call host work of building
    the call and launching each kernel) and returns the static output (overwritten by the next
    call).

    host_io=True also captures the transfers: the graph copies x and logits from pinned host
    buffers (`x_host`, `logits_host`) to the device, runs the layer and copies the output back
    to a pinned host buffer (`out_host`), so one replay is the whole host-to-host step.  Fill
    the host inputs in place (or pass host tensors, which are first copied into them on the
    CPU); the returned `out_host` is valid once the current stream has reached the replay's
    end (e.g. after torch.cuda.current_stream().synchronize())."""

    def __init__(self, layer: MoeFFN, T: int, host_io: bool = False):
        dev = layer.w.w13_codes.device
        self.layer, self.T, self.host_io = layer, T, host_io
        self.x = torch.zeros(T, layer.w.H, dtype=torch.bfloat16, device=dev)
        self.logits = torch.zeros(T, layer.w.E, dtype=torch.float32, device=dev)
        self.out = torch.empty(T, layer.w.H, dtype=torch.bfloat16, device=dev)
        if host_io:
            self.x_host = torch.zeros(T, layer.w.H, dtype=torch.bfloat16).pin_memory()
            self.logits_host = torch.zeros(T, layer.w.E, dtype=torch.float32).pin_memory()
            self.out_host = torch.empty(T, layer.w.H, dtype=torch.bfloat16).pin_memory()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            layer(self.x, self.logits, out=self.out)  # workspace and kernel attributes set up
        torch.cuda.current_stream(dev).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            if host_io:
                self.x.copy_(self.x_host, non_blocking=True)
                self.logits.copy_(self.logits_host, non_blocking=True)
            layer(self.x, self.logits, out=self.out)
            if host_io:
                self.out_host.copy_(self.out, non_blocking=True)

    def __call__(self, x: torch.Tensor = None, logits: torch.Tensor = None) -> torch.Tensor:
        if self.host_io:
            for src, dst in ((x, self.x_host), (logits, self.logits_host)):
                if src is not None and src.data_ptr() != dst.data_ptr():
                    if src.shape != dst.shape or src.dtype != dst.dtype or src.is_cuda:
                        raise ValueError(f"host_io takes host {dst.dtype} {tuple(dst.shape)} inputs")
                    dst.copy_(src)
            self.graph.replay()
            return self.out_host
        if x is None or logits is None:
            raise ValueError("x and logits are required")
        if x.shape != self.x.shape or logits.shape != self.logits.shape:
            raise ValueError(f"captured for x {tuple(self.x.shape)}, logits {tuple(self.logits.shape)}")
        self.x.copy_(x, non_blocking=True)
        self.logits.copy_(logits, non_blocking=True)
        self.graph.replay()
        return self.out


def moe_ffn_forward(layer: MoeFFN, x: torch.Tensor, logits: torch.Tensor, **kw) -> torch.Tensor:
    return layer.forward(x, logits, **kw)
