"""The quantiser entry point for callers that cannot allocate device memory.

nvfp4_quantize_dynamic_noalloc exists for code that may not call cudaMalloc and has no
workspace to pass (for example a plug-in inside a host framework that owns the device
allocator, or a deployment with a fixed device-memory budget).  It keeps its scratch in a
64 KiB array compiled into the library.  These tests call it through the C ABI and check
that it produces exactly what the workspace-taking entry point produces, on two calls in a
row (the second call finds the first call's leftovers in the shared scratch), and that a
size needing more scratch than the array holds is refused with a clear error.

This file is collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from nvfp4_mixture_experts_w4a4_b200 import _lib as C
from nvfp4_mixture_experts_w4a4_b200 import ops
from tests.helpers import layouts as LY

pytestmark = pytest.mark.gpu


def _noalloc(x: torch.Tensor, sf_layout: int):
    B, rows, K = x.shape
    codes = torch.empty(B, rows, K // 2, dtype=torch.uint8, device=x.device)
    sfb = ops.sf_mma_bytes(rows, K) if sf_layout == C.SF_MMA else rows * (K // 16)
    sf = torch.empty(B, sfb, dtype=torch.uint8, device=x.device)
    scale = torch.empty(B, dtype=torch.float32, device=x.device)
    dt = C.DTYPE_BF16 if x.dtype == torch.bfloat16 else C.DTYPE_F32
    st = C.lib().nvfp4_quantize_dynamic_noalloc(
        ctypes.c_void_p(x.data_ptr()), dt, B, rows, K, x.stride(1), x.stride(0), None, rows,
        ctypes.c_void_p(scale.data_ptr()), ctypes.c_void_p(codes.data_ptr()), codes.stride(0),
        ctypes.c_void_p(sf.data_ptr()), sf.stride(0), sf_layout,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    C.check(st, "nvfp4_quantize_dynamic_noalloc")
    return codes, sf, scale


def _inputs(seed: int, B: int, rows: int, K: int, dtype):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, rows, K, generator=g)
    x[:, :, ::37] *= 30.0          # outlier channels
    x[0, 0, :16] = 0.0             # a zero block
    return x.to(dtype).cuda()


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        raise RuntimeError("this test needs a CUDA device")
    # the first call leaves many partials in the shared scratch; the second reads fewer
    for seed, (B, rows, K, dtype, layout) in enumerate([(4, 1000, 2048, torch.bfloat16, C.SF_MMA),
                                                         (1, 37, 512, torch.float32, C.SF_ROWMAJOR)]):
        x = _inputs(seed + 1, B, rows, K, dtype)
        ref_codes, ref_sf, ref_scale = ops.nvfp4_quantize(x, None, sf_layout=layout)
        codes, sf, scale = _noalloc(x, layout)
        torch.cuda.synchronize()
        assert torch.equal(scale, ref_scale)
        assert torch.equal(codes, ref_codes)
        # compare the scales of the real rows only (the MMA layout pads rows to 128)
        for b in range(B):
            got, ref = sf[b].cpu().numpy(), ref_sf[b].cpu().numpy()
            if layout == C.SF_MMA:
                got, ref = LY.from_mma(got, rows, K), LY.from_mma(ref, rows, K)
            assert np.array_equal(got, ref)
        assert np.isfinite(scale.cpu().numpy()).all() and (scale > 0).all()


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # 40 matrices of 4096 x 2048 need 40 * 512 partials = 80 KiB of scratch (> 64 KiB);
    # the size check runs before any pointer is used
    st = C.lib().nvfp4_quantize_dynamic_noalloc(None, C.DTYPE_BF16, 40, 4096, 2048, 2048, 4096 * 2048, None,
                                                4096, None, None, 0, None, 0, C.SF_MMA, None)
    assert st == C.UNSUPPORTED_SHAPE
    msg = C.lib().nvfp4moe_last_error().decode()
    assert "81920 bytes of scratch" in msg and "65536" in msg
