"""CPU oracle for the NVFP4 W4A4 routed-MoE feed-forward layer (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path never does.  The arithmetic lives in
``nvfp4_oracle.cpp`` (see its header for the readings R1..R9 of the pages); this module is
argument marshalling over ctypes and numpy.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)


class MoeArgs(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
        ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("nthreads", ctypes.c_int32),
        ("x_bf16", _u16p), ("logits", _f32p),
        ("x_scale_mode", ctypes.c_int32), ("x_scale", _f32p),
        ("wg_codes", _u8p), ("wg_sf", _u8p), ("wg_scale", _f32p),
        ("wu_codes", _u8p), ("wu_sf", _u8p), ("wu_scale", _f32p),
        ("wd_codes", _u8p), ("wd_sf", _u8p), ("wd_scale", _f32p),
        ("h_scale_mode", ctypes.c_int32), ("h_scale", _f32p),
        ("out_bf16", _u16p), ("out_f64", _f64p),
        ("ids", _i32p), ("w", _f32p), ("counts", _i32p), ("offsets", _i32p),
        ("row_token", _i32p), ("row_slot", _i32p), ("pair_to_row", _i32p),
        ("x_codes", _u8p), ("x_sf", _u8p), ("h_f32", _f32p), ("h_codes", _u8p),
        ("h_sf", _u8p), ("h_amax", _f32p), ("y_f64", _f64p),
        ("shared_I", ctypes.c_int32), ("shared_g", _u16p), ("shared_u", _u16p), ("shared_d", _u16p),
    ]


class MoeW4A16Args(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
        ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("nthreads", ctypes.c_int32),
        ("x_bf16", _u16p), ("logits", _f32p),
        ("wg_codes", _u8p), ("wg_sf", _u8p), ("wg_scale", _f32p),
        ("wu_codes", _u8p), ("wu_sf", _u8p), ("wu_scale", _f32p),
        ("wd_codes", _u8p), ("wd_sf", _u8p), ("wd_scale", _f32p),
        ("out_bf16", _u16p), ("out_f64", _f64p),
        ("ids", _i32p), ("w", _f32p), ("counts", _i32p), ("offsets", _i32p),
        ("row_token", _i32p), ("pair_to_row", _i32p), ("h_bf16", _u16p), ("y_f64", _f64p),
        ("shared_I", ctypes.c_int32), ("shared_g", _u16p), ("shared_u", _u16p), ("shared_d", _u16p),
    ]


def _declare(L):
    L.orc_e2m1_value.restype = ctypes.c_double
    L.orc_e2m1_value.argtypes = [ctypes.c_int]
    L.orc_e2m1_encode.restype = ctypes.c_int
    L.orc_e2m1_encode.argtypes = [ctypes.c_float]
    L.orc_e4m3_value.restype = ctypes.c_double
    L.orc_e4m3_value.argtypes = [ctypes.c_int]
    L.orc_e4m3_encode.restype = ctypes.c_int
    L.orc_e4m3_encode.argtypes = [ctypes.c_float]
    L.orc_float_to_bf16.restype = ctypes.c_uint16
    L.orc_float_to_bf16.argtypes = [ctypes.c_float]
    L.orc_e2m1_encode_n.restype = None
    L.orc_e2m1_encode_n.argtypes = [_f32p, ctypes.c_int64, _u8p]
    L.orc_e4m3_encode_n.restype = None
    L.orc_e4m3_encode_n.argtypes = [_f32p, ctypes.c_int64, _u8p]
    L.orc_quantize.restype = ctypes.c_int
    L.orc_quantize.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, _f32p,
                               _u8p, _u8p]
    L.orc_dequantize.restype = None
    L.orc_dequantize.argtypes = [_u8p, _u8p, ctypes.c_float, ctypes.c_int64, ctypes.c_int64,
                                 _f64p]
    L.orc_gemm.restype = None
    L.orc_gemm.argtypes = [_u8p, _u8p, ctypes.c_float, _u8p, _u8p, ctypes.c_float,
                           ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _f64p, ctypes.c_int]
    L.orc_route.restype = None
    L.orc_route.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _f32p]
    L.orc_permute.restype = ctypes.c_int
    L.orc_permute.argtypes = [_i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _i32p,
                              _i32p, _i32p, _i32p]
    L.orc_moe_ffn.restype = ctypes.c_int
    L.orc_moe_ffn.argtypes = [ctypes.POINTER(MoeArgs)]
    L.orc_e8m0_value.restype = ctypes.c_double
    L.orc_e8m0_value.argtypes = [ctypes.c_int]
    L.orc_mx_quantize.restype = ctypes.c_int
    L.orc_mx_quantize.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int64, _u8p, _u8p]
    L.orc_mx_dequantize.restype = None
    L.orc_mx_dequantize.argtypes = [_u8p, _u8p, ctypes.c_int64, ctypes.c_int64, _f64p]
    L.orc_mx_to_nvfp4.restype = ctypes.c_int
    L.orc_mx_to_nvfp4.argtypes = [_u8p, _u8p, ctypes.c_int64, ctypes.c_int64, _u8p, _f32p]
    L.orc_moe_ffn_w4a16.restype = ctypes.c_int
    L.orc_moe_ffn_w4a16.argtypes = [ctypes.POINTER(MoeW4A16Args)]


def _p(a: np.ndarray | None, ctype):
    if a is None:
        return ctypes.cast(None, ctypes.POINTER(ctype))
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


# ------------------------------------------------------------------ codec ----
def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e2m1_encode(q: float) -> int:
    return lib().orc_e2m1_encode(float(q))


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(int(code))


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(float(v))


def e2m1_encode_array(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, np.float32).ravel()
    out = np.zeros(q.size, np.uint8)
    lib().orc_e2m1_encode_n(_p(q, ctypes.c_float), q.size, _p(out, ctypes.c_uint8))
    return out


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32).ravel()
    out = np.zeros(v.size, np.uint8)
    lib().orc_e4m3_encode_n(_p(v, ctypes.c_float), v.size, _p(out, ctypes.c_uint8))
    return out


def float_to_bf16(f: float) -> int:
    return lib().orc_float_to_bf16(float(f))


# -------------------------------------------------------------- quantiser ----
def quantize(x: np.ndarray, tensor_scale: float | None = None):
    """Quantise a row-major fp32 matrix [rows, K] to NVFP4.

    tensor_scale None -> dynamic (amax / 2688).  Returns (codes [rows, K/2] u8,
    sf [rows, K/16] u8 E4M3 codes, row-major, tensor scale as float).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, K = x.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    sf = np.zeros((rows, K // 16), np.uint8)
    ts = np.array([0.0 if tensor_scale is None else tensor_scale], np.float32)
    rc = lib().orc_quantize(_p(x, ctypes.c_float), rows, K, 1 if tensor_scale is None else 0,
                            _p(ts, ctypes.c_float), _p(codes, ctypes.c_uint8),
                            _p(sf, ctypes.c_uint8))
    if rc != 0:
        raise ValueError("orc_quantize: K must be a multiple of 16")
    return codes, sf, float(ts[0])


def dequantize(codes: np.ndarray, sf: np.ndarray, tensor_scale: float) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    sf = np.ascontiguousarray(sf, np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((rows, K), np.float64)
    lib().orc_dequantize(_p(codes, ctypes.c_uint8), _p(sf, ctypes.c_uint8), tensor_scale, rows, K,
                         _p(out, ctypes.c_double))
    return out


def gemm(a_codes, a_sf, s_a, b_codes, b_sf, s_b, nthreads: int | None = None) -> np.ndarray:
    """C = A @ B^T of two NVFP4 matrices (both K-major), exact blocks, fp64."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_sf = np.ascontiguousarray(a_sf, np.uint8)
    b_sf = np.ascontiguousarray(b_sf, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    out = np.zeros((M, N), np.float64)
    lib().orc_gemm(_p(a_codes, ctypes.c_uint8), _p(a_sf, ctypes.c_uint8), s_a,
                   _p(b_codes, ctypes.c_uint8), _p(b_sf, ctypes.c_uint8), s_b, M, N, K,
                   _p(out, ctypes.c_double), nthreads or default_threads())
    return out


# --------------------------------------------------------- route, permute ----
def route(logits: np.ndarray, k: int):
    logits = np.ascontiguousarray(logits, np.float32)
    T, E = logits.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    lib().orc_route(_p(logits, ctypes.c_float), T, E, k, _p(ids, ctypes.c_int32),
                    _p(w, ctypes.c_float))
    return ids, w


def permute(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, np.int32)
    T, k = ids.shape
    P = T * k
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    row_token = np.zeros(P, np.int32)
    row_slot = np.zeros(P, np.int32)
    pair_to_row = np.zeros(P, np.int32)
    rc = lib().orc_permute(_p(ids, ctypes.c_int32), T, E, k, _p(counts, ctypes.c_int32),
                           _p(offsets, ctypes.c_int32), _p(row_token, ctypes.c_int32),
                           _p(row_slot, ctypes.c_int32), _p(pair_to_row, ctypes.c_int32))
    if rc != 0:
        raise ValueError("orc_permute: expert id out of range")
    return dict(counts=counts, offsets=offsets, row_token=row_token, row_slot=row_slot,
                pair_to_row=pair_to_row)


# ------------------------------------------------------------------ layer ----
def quantize_experts(w: np.ndarray):
    """Quantise stacked per-expert fp32 weights [E, N, K] with one dynamic tensor scale per
    expert.  Returns codes [E, N, K/2], sf [E, N, K/16] (row-major), scale [E] fp32."""
    E, N, K = w.shape
    codes = np.zeros((E, N, K // 2), np.uint8)
    sf = np.zeros((E, N, K // 16), np.uint8)
    sc = np.zeros(E, np.float32)
    for e in range(E):
        c, s, t = quantize(w[e])
        codes[e], sf[e], sc[e] = c, s, t
    return codes, sf, sc


def _set_shared(a, shared, keep: list):
    """shared: None or (g [I_s, H], u [I_s, H], d [H, I_s]) bf16 bit patterns (reading R12)."""
    if shared is None:
        a.shared_I = 0
        return
    g, u, d = (np.ascontiguousarray(v, np.uint16) for v in shared)
    keep += [g, u, d]
    a.shared_I = g.shape[0]
    a.shared_g, a.shared_u, a.shared_d = (_p(v, ctypes.c_uint16) for v in (g, u, d))


def moe_ffn(x_bf16: np.ndarray, logits: np.ndarray, k: int, wg, wu, wd, *, x_scale=None,
            h_scale=None, nthreads: int | None = None, want_y: bool = False, shared=None) -> dict:
    """Runs the whole layer on the CPU.

    x_bf16: uint16 [T, H] bf16 bit patterns; logits fp32 [T, E];
    wg, wu: (codes [E, I, H/2], sf [E, I, H/16], scale [E]); wd: (codes [E, H, I/2],
    sf [E, H, I/16], scale [E]).  x_scale None -> dynamic.  h_scale None -> calibrate
    (amax of each expert's h / 2688), else fp32 [E] given.
    Returns a dict with out_bf16 (uint16 [T, H]), out_f64 and every intermediate.
    """
    x_bf16 = np.ascontiguousarray(x_bf16, np.uint16)
    logits = np.ascontiguousarray(logits, np.float32)
    T, H = x_bf16.shape
    E = logits.shape[1]
    I = wg[0].shape[1]
    P = T * k
    wg = [np.ascontiguousarray(v) for v in wg]
    wu = [np.ascontiguousarray(v) for v in wu]
    wd = [np.ascontiguousarray(v) for v in wd]
    xs = np.array([0.0 if x_scale is None else x_scale], np.float32)
    hs = (np.zeros(E, np.float32) if h_scale is None
          else np.ascontiguousarray(h_scale, np.float32).copy())
    r = dict(
        out_bf16=np.zeros((T, H), np.uint16), out_f64=np.zeros((T, H), np.float64),
        ids=np.zeros((T, k), np.int32), w=np.zeros((T, k), np.float32),
        counts=np.zeros(E, np.int32), offsets=np.zeros(E + 1, np.int32),
        row_token=np.zeros(P, np.int32), row_slot=np.zeros(P, np.int32),
        pair_to_row=np.zeros(P, np.int32),
        x_codes=np.zeros((T, H // 2), np.uint8), x_sf=np.zeros((T, H // 16), np.uint8),
        h_f32=np.zeros((P, I), np.float32), h_codes=np.zeros((P, I // 2), np.uint8),
        h_sf=np.zeros((P, I // 16), np.uint8), h_amax=np.zeros(E, np.float32),
        y_f64=np.zeros((P, H), np.float64) if want_y else None,
    )
    a = MoeArgs()
    a.T, a.H, a.I, a.E, a.k = T, H, I, E, k
    a.nthreads = nthreads or default_threads()
    a.x_bf16 = _p(x_bf16, ctypes.c_uint16)
    a.logits = _p(logits, ctypes.c_float)
    a.x_scale_mode = 1 if x_scale is None else 0
    a.x_scale = _p(xs, ctypes.c_float)
    a.wg_codes, a.wg_sf, a.wg_scale = (_p(wg[0], ctypes.c_uint8), _p(wg[1], ctypes.c_uint8),
                                       _p(wg[2], ctypes.c_float))
    a.wu_codes, a.wu_sf, a.wu_scale = (_p(wu[0], ctypes.c_uint8), _p(wu[1], ctypes.c_uint8),
                                       _p(wu[2], ctypes.c_float))
    a.wd_codes, a.wd_sf, a.wd_scale = (_p(wd[0], ctypes.c_uint8), _p(wd[1], ctypes.c_uint8),
                                       _p(wd[2], ctypes.c_float))
    a.h_scale_mode = 1 if h_scale is None else 0
    a.h_scale = _p(hs, ctypes.c_float)
    a.out_bf16 = _p(r["out_bf16"], ctypes.c_uint16)
    a.out_f64 = _p(r["out_f64"], ctypes.c_double)
    for name, ct in (("ids", ctypes.c_int32), ("w", ctypes.c_float), ("counts", ctypes.c_int32),
                     ("offsets", ctypes.c_int32), ("row_token", ctypes.c_int32),
                     ("row_slot", ctypes.c_int32), ("pair_to_row", ctypes.c_int32),
                     ("x_codes", ctypes.c_uint8), ("x_sf", ctypes.c_uint8),
                     ("h_f32", ctypes.c_float), ("h_codes", ctypes.c_uint8),
                     ("h_sf", ctypes.c_uint8), ("h_amax", ctypes.c_float),
                     ("y_f64", ctypes.c_double)):
        setattr(a, name, _p(r[name], ct))
    # keep every buffer alive for the duration of the call
    keep = [x_bf16, logits, wg, wu, wd, xs, hs, r]
    _set_shared(a, shared, keep)
    rc = lib().orc_moe_ffn(ctypes.byref(a))
    del keep
    if rc != 0:
        raise ValueError(f"orc_moe_ffn failed ({rc})")
    r["x_scale"] = float(xs[0])
    r["h_scale"] = hs
    return r


def moe_ffn_w4a16(x_bf16: np.ndarray, logits: np.ndarray, k: int, wg, wu, wd, *,
                  nthreads: int | None = None, want_y: bool = False, shared=None) -> dict:
    """The weight-only (W4A16) layer on the CPU (reading R10 of nvfp4_oracle.cpp): bf16 x
    into the gate/up products, h rounded to bf16, NVFP4 weights dequantised, fp64 sums.
    Arguments as for moe_ffn.  Returns out_bf16, out_f64, the routing and permutation, and
    h_bf16 (uint16 [T*k, I], permuted rows)."""
    x_bf16 = np.ascontiguousarray(x_bf16, np.uint16)
    logits = np.ascontiguousarray(logits, np.float32)
    T, H = x_bf16.shape
    E = logits.shape[1]
    I = wg[0].shape[1]
    P = T * k
    wg = [np.ascontiguousarray(v) for v in wg]
    wu = [np.ascontiguousarray(v) for v in wu]
    wd = [np.ascontiguousarray(v) for v in wd]
    r = dict(
        out_bf16=np.zeros((T, H), np.uint16), out_f64=np.zeros((T, H), np.float64),
        ids=np.zeros((T, k), np.int32), w=np.zeros((T, k), np.float32),
        counts=np.zeros(E, np.int32), offsets=np.zeros(E + 1, np.int32),
        row_token=np.zeros(P, np.int32), pair_to_row=np.zeros(P, np.int32),
        h_bf16=np.zeros((P, I), np.uint16),
        y_f64=np.zeros((P, H), np.float64) if want_y else None,
    )
    a = MoeW4A16Args()
    a.T, a.H, a.I, a.E, a.k = T, H, I, E, k
    a.nthreads = nthreads or default_threads()
    a.x_bf16 = _p(x_bf16, ctypes.c_uint16)
    a.logits = _p(logits, ctypes.c_float)
    a.wg_codes, a.wg_sf, a.wg_scale = (_p(wg[0], ctypes.c_uint8), _p(wg[1], ctypes.c_uint8),
                                       _p(wg[2], ctypes.c_float))
    a.wu_codes, a.wu_sf, a.wu_scale = (_p(wu[0], ctypes.c_uint8), _p(wu[1], ctypes.c_uint8),
                                       _p(wu[2], ctypes.c_float))
    a.wd_codes, a.wd_sf, a.wd_scale = (_p(wd[0], ctypes.c_uint8), _p(wd[1], ctypes.c_uint8),
                                       _p(wd[2], ctypes.c_float))
    for name, ct in (("out_bf16", ctypes.c_uint16), ("out_f64", ctypes.c_double),
                     ("ids", ctypes.c_int32), ("w", ctypes.c_float), ("counts", ctypes.c_int32),
                     ("offsets", ctypes.c_int32), ("row_token", ctypes.c_int32),
                     ("pair_to_row", ctypes.c_int32), ("h_bf16", ctypes.c_uint16),
                     ("y_f64", ctypes.c_double)):
        setattr(a, name, _p(r[name], ct))
    keep = [x_bf16, logits, wg, wu, wd, r]
    _set_shared(a, shared, keep)
    rc = lib().orc_moe_ffn_w4a16(ctypes.byref(a))
    del keep
    if rc != 0:
        raise ValueError(f"orc_moe_ffn_w4a16 failed ({rc})")
    return r


# ------------------------------------------------------------------ MXFP4 (R11) ----
def e8m0_value(code: int) -> float:
    return lib().orc_e8m0_value(int(code))


def mx_quantize(x: np.ndarray):
    """MXFP4 quantisation of fp32 [rows, K] (K % 32 == 0): codes [rows, K/2] u8 and E8M0
    scales [rows, K/32] u8."""
    x = np.ascontiguousarray(x, np.float32)
    rows, K = x.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    e8m0 = np.zeros((rows, K // 32), np.uint8)
    if lib().orc_mx_quantize(_p(x, ctypes.c_float), rows, K, _p(codes, ctypes.c_uint8), _p(e8m0, ctypes.c_uint8)):
        raise ValueError("orc_mx_quantize: K must be a multiple of 32")
    return codes, e8m0


def mx_dequantize(codes: np.ndarray, e8m0: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    e8m0 = np.ascontiguousarray(e8m0, np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((rows, K), np.float64)
    lib().orc_mx_dequantize(_p(codes, ctypes.c_uint8), _p(e8m0, ctypes.c_uint8), rows, K, _p(out, ctypes.c_double))
    return out


def mx_to_nvfp4(codes: np.ndarray, e8m0: np.ndarray):
    """The exact NVFP4 form of an MXFP4 matrix: (codes unchanged, row-major E4M3 scales
    [rows, K/16], tensor scale).  Raises ValueError when no exact form exists."""
    codes = np.ascontiguousarray(codes, np.uint8)
    e8m0 = np.ascontiguousarray(e8m0, np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    sf = np.zeros((rows, K // 16), np.uint8)
    ts = np.zeros(1, np.float32)
    rc = lib().orc_mx_to_nvfp4(_p(codes, ctypes.c_uint8), _p(e8m0, ctypes.c_uint8), rows, K, _p(sf, ctypes.c_uint8),
                               _p(ts, ctypes.c_float))
    if rc:
        raise ValueError(f"orc_mx_to_nvfp4 failed ({rc})")
    return codes, sf, float(ts[0])


def mx_experts_to_nvfp4(codes: np.ndarray, e8m0: np.ndarray):
    """mx_to_nvfp4 per expert of stacked [E, N, ...] arrays: (codes, sf [E, N, K/16], scale [E])."""
    E = codes.shape[0]
    sf = np.zeros(codes.shape[:2] + (codes.shape[2] // 8,), np.uint8)
    sc = np.zeros(E, np.float32)
    for e in range(E):
        _, sf[e], sc[e] = mx_to_nvfp4(codes[e], e8m0[e])
    return codes, sf, sc
