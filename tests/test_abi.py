"""Host-side checks of the C ABI (no GPU needed): the library builds, loads, exports every
function that include/*.h declares, the binding declares each of them, and argument
errors come back as status codes with a message before anything is launched."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                             src, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def so():
    from nvfp4_mixture_experts_w4a4_b200 import build, _lib
    path = build.build()
    assert os.path.samefile(path, _lib.LIB_PATH)
    return _lib.lib()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for fn in ("nvfp4_quantize", "moe_route", "moe_permute", "moe_ffn_forward", "nvfp4_gemm"):
        assert fn in names


def test_library_exports_every_declared_symbol(so):
    for fn in sorted(_declared_functions()):
        assert hasattr(so, fn), f"{fn} declared in include/ but not exported"


def test_binding_declares_every_symbol():
    from nvfp4_mixture_experts_w4a4_b200 import _lib
    assert _declared_functions() == set(_lib.SIGNATURES)


def test_argument_errors_are_statuses(so):
    from nvfp4_mixture_experts_w4a4_b200 import _lib as C
    assert so.nvfp4moe_version() == 0x000600
    # bad E, bad k: rejected before any device work
    assert so.moe_route(None, 4, 2000, 2, None, None, None) == C.UNSUPPORTED_SHAPE
    assert b"E=2000" in so.nvfp4moe_last_error()
    assert so.moe_route(None, 4, 8, 9, None, None, None) == C.UNSUPPORTED_SHAPE
    assert so.moe_route(None, 4, 8, 2, None, None, None) == C.INVALID_ARG
    # quantiser: K not a multiple of 16, MMA layout with K % 64 != 0
    assert so.nvfp4_quantize(None, 0, 1, 4, 24, 24, 0, None, 4, 0, None, None, 0, None, 0, 0, None, 0,
                             None) == C.UNSUPPORTED_SHAPE
    assert so.nvfp4_quantize(None, 0, 1, 4, 32, 32, 0, None, 4, 0, None, None, 0, None, 0, 1, None, 0,
                             None) == C.UNSUPPORTED_SHAPE
    assert so.nvfp4_quantize(None, 7, 1, 4, 32, 32, 0, None, 4, 0, None, None, 0, None, 0, 0, None, 0,
                             None) == C.INVALID_ARG
    # empty work is a no-op success
    assert so.moe_route(None, 0, 8, 2, None, None, None) == C.OK
    assert so.nvfp4_gemm(None, None, None, None, None, None, 0, 128, 256, None, 0, None, 0, None) == C.OK
    assert so.nvfp4_gemm(None, None, None, None, None, None, 4, 128, 192, None, 0, None, 0, None) == \
        C.UNSUPPORTED_SHAPE
    assert so.nvfp4_gemm(None, None, None, None, None, None, 4, 100, 256, None, 0, None, 0, None) == \
        C.UNSUPPORTED_SHAPE
    # weight preparation: K % 64, unknown layouts, out_rows without a gather, codes_out without codes
    assert so.nvfp4_prep_weights(None, None, 0, 1, 4, 96, None, 4, None, None, 1, None) == C.UNSUPPORTED_SHAPE
    assert so.nvfp4_prep_weights(None, None, 2, 1, 4, 64, None, 4, None, None, 1, None) == C.INVALID_ARG
    assert so.nvfp4_prep_weights(None, None, 0, 1, 4, 64, None, 8, None, None, 1, None) == C.INVALID_ARG
    assert so.nvfp4_prep_weights(None, 64, 0, 1, 4, 64, None, 4, 128, 128, 1, None) == C.INVALID_ARG
    assert so.nvfp4_prep_weights(None, None, 0, 0, 4, 64, None, 4, None, None, 1, None) == C.OK


def test_workspace_queries(so):
    from nvfp4_mixture_experts_w4a4_b200 import _lib as C
    d = C.MoeFfnDesc()
    d.T, d.H, d.I, d.E, d.top_k = 16, 2048, 512, 512, 10
    d.x_scale_mode = C.SCALE_DYNAMIC
    L = C.MoeFfnWsLayout()
    assert so.moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L)) == C.OK
    # no GPU here: the tensor-core path is unavailable, AUTO falls back to the GEMV layout
    assert L.path == C.PATH_GEMV and L.m_tile == 1
    assert so.moe_ffn_workspace_size(ctypes.byref(d)) == L.total > 0
    offs = sorted([L.topk_ids, L.topk_w, L.counts, L.offsets, L.padded_offsets, L.pair_to_row, L.row_token,
                   L.row_pair, L.tile_expert, L.active, L.x_scale, L.x_codes, L.x_sf, L.h_codes, L.h_sf,
                   L.slots])
    assert all(o % 256 == 0 for o in offs) and len(set(offs)) == len(offs) and offs[-1] < L.total
    # launch modes: every named one is accepted (on this host none can take the single launch,
    # which needs the tensor-core path), anything else is an argument error
    for mode in (C.LAUNCH_AUTO, C.LAUNCH_SINGLE, C.LAUNCH_MULTI, C.LAUNCH_SINGLE_TILE, C.LAUNCH_SINGLE_LOCAL):
        d.launch_mode = mode
        assert so.moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L)) == C.OK
        assert L.single_launch == 0
    for bad in (-1, 5):
        d.launch_mode = bad
        assert so.moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L)) == C.INVALID_ARG
    d.launch_mode = C.LAUNCH_AUTO
    d.H = 100
    assert so.moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L)) == C.UNSUPPORTED_SHAPE
    assert so.moe_permute_rows_capacity(16, 512, 10, 128) == 160 + 160 * 127
    assert so.moe_permute_rows_capacity(4096, 256, 8, 128) == 32768 + 256 * 127


def test_weight_only_workspace_and_mode_checks(so):
    """The weight-only (W4A16) mode: no activation codes in the workspace, a bf16 h region,
    the GEMV path whatever AUTO would pick, and the tensor-core path or a bad mode refused."""
    from nvfp4_mixture_experts_w4a4_b200 import _lib as C
    d = C.MoeFfnDesc()
    d.T, d.H, d.I, d.E, d.top_k = 16, 2048, 512, 512, 10
    d.act_mode = C.ACT_BF16
    L = C.MoeFfnWsLayout()
    assert so.moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L)) == C.OK
    assert L.path == C.PATH_GEMV and L.x_rows == 0 and L.h_rows == 0
    assert L.h_bf16 % 256 == 0 and L.h_bf16 + 16 * 10 * 512 * 2 <= L.total
    d.path = C.PATH_GEMM
    assert so.moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L)) == C.UNSUPPORTED_SHAPE
    d.path, d.act_mode = C.PATH_AUTO, 7
    assert so.moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L)) == C.INVALID_ARG


@pytest.mark.parametrize("path", [0, 1, 2])
@pytest.mark.parametrize("act", [0, 1])
@pytest.mark.parametrize("shared_I", [0, 128])
def test_workspace_layout_of_an_empty_batch(so, path, act, shared_I):
    """T = 0 lays out a workspace (no division by the empty batch) on every path and mode."""
    from nvfp4_mixture_experts_w4a4_b200 import _lib as C
    d = C.MoeFfnDesc()
    d.T, d.H, d.I, d.E, d.top_k = 0, 256, 128, 8, 2
    d.path, d.act_mode, d.shared_I = path, act, shared_I
    L = C.MoeFfnWsLayout()
    st = so.moe_ffn_workspace_layout(ctypes.byref(d), ctypes.byref(L))
    assert st == (C.UNSUPPORTED_SHAPE if (act == 1 and path == 2) else C.OK)


C_CLIENT = r"""
/* A plain C99 client of the boundary: the header must compile as C, and argument errors
   come back as status codes (no device is touched). */
#include <stdio.h>
#include <string.h>
#include "nvfp4moe.h"

int main(void) {
  moe_ffn_desc d;
  memset(&d, 0, sizeof d);
  d.T = 4; d.H = 100; d.I = 128; d.E = 8; d.top_k = 2;      /* H not a multiple of 64 */
  if (nvfp4moe_version() != 0x000600) return 1;
  if (moe_ffn_workspace_size(&d) != 0) return 2;             /* an invalid desc needs nothing */
  if (moe_route(NULL, 4, 8, 9, NULL, NULL, NULL) != NVFP4MOE_UNSUPPORTED_SHAPE) return 3;
  if (strstr(nvfp4moe_last_error(), "k=9") == NULL) return 4;
  if (nvfp4_prep_weights(NULL, NULL, NVFP4MOE_SF_ROWMAJOR, 0, 4, 64, NULL, 4, NULL, NULL, NVFP4MOE_SF_MMA,
                         NULL) != NVFP4MOE_OK) return 5;       /* an empty batch is a no-op */
  printf("ok\n");
  return 0;
}
"""


def test_header_compiles_as_c99_and_links(so):
    """The boundary as a C program sees it: include/nvfp4moe.h compiles with a C compiler in
    strict C99, and a program linked against libnvfp4moe.so gets status codes and messages."""
    import subprocess
    from nvfp4_mixture_experts_w4a4_b200 import _lib
    work = os.path.join(ROOT, "_build", "c_client")
    os.makedirs(work, exist_ok=True)
    src, exe = os.path.join(work, "client.c"), os.path.join(work, "client")
    with open(src, "w") as f:
        f.write(C_CLIENT)
    libdir = os.path.dirname(_lib.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                         src, "-o", exe, "-L", libdir, "-l:libnvfp4moe.so", "-Wl,-rpath," + libdir],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)
