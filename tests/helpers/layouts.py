"""Test-side (numpy) conversions between the oracle's canonical layouts and the library's
device layouts.  Written from the layout definitions in include/nvfp4moe.h, independently
of the CUDA sources.
"""
import numpy as np


def sf_mma_bytes(rows: int, K: int) -> int:
    return ((rows + 127) // 128) * 128 * (K // 16)


def _mma_index(rows: int, K: int):
    r = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    return ((r // 128) * (K // 64) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4


def to_mma(sf: np.ndarray, K: int) -> np.ndarray:
    """Row-major scales [rows, K/16] -> MMA-layout bytes (padding rows zero)."""
    rows = sf.shape[0]
    out = np.zeros(sf_mma_bytes(rows, K), np.uint8)
    out[_mma_index(rows, K)] = sf
    return out


def from_mma(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """MMA-layout bytes -> row-major scales [rows, K/16]."""
    return np.asarray(buf).reshape(-1)[_mma_index(rows, K)]


def interleave_rows(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """[I, X] gate and up -> [2I, X] with W13 row 32c+j = gate 16c+j (j<16), up 16c+j-16."""
    I = gate.shape[0]
    out = np.empty((2 * I,) + gate.shape[1:], gate.dtype)
    g = gate.reshape(I // 16, 16, *gate.shape[1:])
    u = up.reshape(I // 16, 16, *up.shape[1:])
    out.reshape(I // 16, 32, *gate.shape[1:])[:, :16] = g
    out.reshape(I // 16, 32, *gate.shape[1:])[:, 16:] = u
    return out


def experts_to_device_layout(wg, wu, wd):
    """Oracle canonical expert weights -> (w13_codes, w13_sf, w13_scale, w2_codes, w2_sf, w2_scale)
    numpy arrays in the library's layout."""
    gc, gs, gsc = wg
    uc, us, usc = wu
    dc, ds, dsc = wd
    E, I, H2 = gc.shape
    H = H2 * 2
    w13_codes = np.stack([interleave_rows(gc[e], uc[e]) for e in range(E)])
    w13_sf = np.stack([to_mma(interleave_rows(gs[e], us[e]), H) for e in range(E)])
    w13_scale = np.stack([gsc, usc], 1).astype(np.float32)
    w2_codes = np.ascontiguousarray(dc)
    w2_sf = np.stack([to_mma(ds[e], I) for e in range(E)])
    return w13_codes, w13_sf, w13_scale, w2_codes, w2_sf, dsc.astype(np.float32)
