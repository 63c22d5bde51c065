"""An independent second formulation of the NVFP4 block quantiser, used only to pin the
oracle.  It is written with numpy fp32 array arithmetic and ml_dtypes' E2M1 / E4M3 casts
(a third-party implementation of the two formats), and shares nothing with the oracle's
C++ encoders.

E4M3 in ml_dtypes turns values above 464 into NaN instead of saturating, so the block
scale ratio is clamped to 448 first (saturate-to-finite).
"""
import ml_dtypes
import numpy as np

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def e2m1_codes_from_values(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, np.float32).astype(F4).view(np.uint8) & 0xF


def e2m1_values_from_codes(c: np.ndarray) -> np.ndarray:
    return (np.asarray(c, np.uint8) & 0xF).view(F4).astype(np.float64)


def e4m3_codes_from_values(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, np.float32)
    v = np.clip(v, np.float32(-448.0), np.float32(448.0))
    return v.astype(F8).view(np.uint8)


def e4m3_values_from_codes(c: np.ndarray) -> np.ndarray:
    return np.asarray(c, np.uint8).view(F8).astype(np.float64)


def quantize(x: np.ndarray, s_t: np.float32):
    """x [rows, K] fp32 -> (codes [rows, K/2], sf [rows, K/16]) with tensor scale s_t."""
    x = np.asarray(x, np.float32)
    rows, K = x.shape
    s_t = np.float32(s_t)
    xb = x.reshape(rows, K // 16, 16)
    amax = np.abs(xb).max(axis=2).astype(np.float32)
    if s_t == 0:
        sf = np.zeros((rows, K // 16), np.uint8)
    else:
        ratio = (amax / (np.float32(6.0) * s_t)).astype(np.float32)
        sf = e4m3_codes_from_values(ratio)
    sfv = e4m3_values_from_codes(sf).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = (np.float32(1.0) / (sfv * s_t).astype(np.float32)).astype(np.float32)
        q = (xb * inv[:, :, None]).astype(np.float32)
    codes = e2m1_codes_from_values(q)
    codes[sfv == 0] = 0
    codes = codes.reshape(rows, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, sf


def dequantize(codes: np.ndarray, sf: np.ndarray, s_t: float) -> np.ndarray:
    codes = np.asarray(codes, np.uint8)
    rows = codes.shape[0]
    K = codes.shape[1] * 2
    lo = e2m1_values_from_codes(codes & 0xF)
    hi = e2m1_values_from_codes(codes >> 4)
    v = np.empty((rows, K), np.float64)
    v[:, 0::2] = lo
    v[:, 1::2] = hi
    sfv = e4m3_values_from_codes(sf)
    return v * np.repeat(sfv, 16, axis=1) * np.float64(s_t)
