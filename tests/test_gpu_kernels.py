"""GPU parity of the individual kernels against the CPU oracle (through the C ABI)."""
import concurrent.futures as cf

import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_mixture_experts_w4a4_b200 import _lib as C
from nvfp4_mixture_experts_w4a4_b200 import ops, workloads as W
from tests import gpu_util as G
from tests.helpers import layouts as LY

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return G.need_gpu()


# ------------------------------------------------------------------ codec ----
def test_codec_every_fp32_bit_pattern(dev):
    """The kernels' E2M1 and E4M3 encoders against the oracle on all 2^32 fp32 patterns
    (NaN inputs excluded: their codes are unspecified)."""
    chunk = 1 << 27
    pool = cf.ThreadPoolExecutor(O.default_threads())
    for start in range(0, 1 << 32, chunk):
        bits = torch.arange(start, start + chunk, dtype=torch.int64, device=dev).to(torch.int32)
        vals = bits.view(torch.float32)
        e2, e4 = ops.codec_convert(vals)
        v = vals.cpu().numpy()
        g2, g4 = e2.cpu().numpy(), e4.cpu().numpy()
        parts = np.array_split(np.arange(v.size), 64)

        def ref(ix):
            return O.e2m1_encode_array(v[ix]), O.e4m3_encode_array(v[ix])

        r = list(pool.map(ref, parts))
        r2 = np.concatenate([a for a, _ in r])
        r4 = np.concatenate([b for _, b in r])
        ok = ~np.isnan(v)
        bad2 = np.nonzero((g2 != r2) & ok)[0]
        bad4 = np.nonzero((g4 != r4) & ok)[0]
        assert bad2.size == 0, (hex(start + int(bad2[0])), v[bad2[0]], g2[bad2[0]], r2[bad2[0]])
        assert bad4.size == 0, (hex(start + int(bad4[0])), v[bad4[0]], g4[bad4[0]], r4[bad4[0]])


# -------------------------------------------------------------- quantiser ----
@pytest.mark.parametrize("rows,K,dtype,given", [
    (1, 64, torch.bfloat16, None), (37, 256, torch.bfloat16, None), (130, 2048, torch.bfloat16, None),
    (129, 320, torch.float32, None), (5, 64, torch.float32, 0.01), (300, 512, torch.bfloat16, 0.5),
])
def test_quantize_parity(dev, rows, K, dtype, given):
    g = torch.Generator().manual_seed(rows * 7 + K)
    x = torch.randn(rows, K, generator=g, dtype=torch.float32)
    x[:, :: max(1, K // 10)] *= 25.0            # outlier channels
    x[min(3, rows - 1), :16] = 0.0              # a zero block
    x[0, 16:32] *= 1e-7                          # an underflowing block
    x = x.to(dtype)
    xf = x.float().numpy()
    rc, rs, rt = O.quantize(xf, tensor_scale=given)
    for layout in (C.SF_MMA, C.SF_ROWMAJOR):
        ts = None if given is None else torch.tensor([given], dtype=torch.float32, device=dev)
        codes, sf, scale = ops.nvfp4_quantize(x.to(dev), ts, sf_layout=layout)
        torch.cuda.synchronize()
        assert scale.item() == np.float32(rt)
        assert np.array_equal(codes.cpu().numpy(), rc)
        sfn = sf.cpu().numpy()
        sfr = LY.from_mma(sfn, rows, K) if layout == C.SF_MMA else sfn.reshape(rows, K // 16)
        assert np.array_equal(sfr, rs)


def test_quantize_batched_gather(dev):
    """Batch of matrices, one dynamic scale each, rows gathered into an interleaved layout
    with skipped rows left untouched (the weight-preparation use)."""
    E, I, H = 3, 64, 256
    g = torch.Generator().manual_seed(11)
    w = torch.randn(E, I, H, generator=g) / 16
    w[1] *= 3.0
    gmap, umap = ops.NVFP4Experts.interleave_maps(I, dev)
    codes = torch.full((E, 2 * I, H // 2), 0xAB, dtype=torch.uint8, device=dev)
    sf = torch.zeros(E, LY.sf_mma_bytes(2 * I, H), dtype=torch.uint8, device=dev)
    _, _, sc = ops.nvfp4_quantize(w.to(dev), None, row_gather=gmap, out_rows=2 * I, codes=codes, sf=sf)
    torch.cuda.synchronize()
    cn, sfn = codes.cpu().numpy(), sf.cpu().numpy()
    for e in range(E):
        rc, rs, rt = O.quantize(w[e].numpy())
        assert sc[e].item() == np.float32(rt)
        gate_rows = np.nonzero(gmap.cpu().numpy() >= 0)[0]
        assert np.array_equal(cn[e][gate_rows], rc)
        assert np.array_equal(LY.from_mma(sfn[e], 2 * I, H)[gate_rows], rs)
        up_rows = np.nonzero(umap.cpu().numpy() >= 0)[0]
        assert (cn[e][up_rows] == 0xAB).all()


def test_quantize_empty_and_errors(dev):
    x = torch.zeros(0, 64, dtype=torch.bfloat16, device=dev)
    codes, sf, _ = ops.nvfp4_quantize(x, torch.ones(1, device=dev))
    assert codes.numel() == 0
    with pytest.raises(C.Nvfp4MoeError):
        ops.nvfp4_quantize(torch.zeros(4, 48, device=dev), None)  # MMA layout needs K % 64


# ---------------------------------------------------------------- routing ----
@pytest.mark.parametrize("T,E,k", [(8, 8, 2), (16, 512, 10), (37, 256, 8), (5, 1024, 32), (3, 1, 1), (64, 33, 32)])
def test_route_parity(dev, T, E, k):
    g = torch.Generator().manual_seed(T * E + k)
    logits = torch.randn(T, E, generator=g)
    logits[0, :] = 0.25                      # all tied
    if T > 1:
        logits[1, ::2] = 0.0
        logits[1, 1::2] = -0.0               # +0 / -0 ties
    if T > 2 and E > 5:
        logits[2, [1, 3, 5]] = 7.0           # tied winners
    ids, w = ops.moe_route(logits.to(dev), k)
    rid, rw = O.route(logits.numpy(), k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)


def test_route_rejects_k_above_32(dev):
    with pytest.raises(C.Nvfp4MoeError, match="k=33"):
        ops.moe_route(torch.zeros(4, 64, device=dev), 33)


# ------------------------------------------------------------ permutation ----
@pytest.mark.parametrize("T,E,k", [(8, 8, 2), (16, 512, 10), (512, 512, 10), (4096, 256, 8), (1, 4, 4), (100, 1, 1),
                                   (33, 1024, 32), (77, 600, 3), (3000, 40, 7)])
@pytest.mark.parametrize("m_tile", [1, 32, 64, 128])
def test_permute_parity(dev, T, E, k, m_tile):
    g = torch.Generator().manual_seed(T + E)
    logits = torch.randn(T, E, generator=g)
    if E > 4:
        logits[:, 3] += 3.0                      # one popular expert
        logits[:, 4] -= 50.0                     # one expert no token picks
    ids, _ = O.route(logits.numpy(), k)
    ref = O.permute(ids, E)
    zero = torch.full((E,), 5.0, device=dev)
    r = ops.moe_permute(torch.from_numpy(ids).to(dev), E, m_tile, zero_f32=zero)
    torch.cuda.synchronize()
    assert (zero == 0).all()
    counts = r["counts"].cpu().numpy()
    assert np.array_equal(counts, ref["counts"])
    assert np.array_equal(r["offsets"].cpu().numpy(), ref["offsets"])
    po = r["padded_offsets"].cpu().numpy()
    assert np.array_equal(po, np.concatenate([[0], np.cumsum((counts + m_tile - 1) // m_tile * m_tile)]))
    p2r = r["pair_to_row"].cpu().numpy()[: T * k]
    e_of_pair = ids.reshape(-1)
    assert np.array_equal(p2r - po[e_of_pair] + ref["offsets"][e_of_pair], ref["pair_to_row"])
    rt, rp = r["row_token"].cpu().numpy(), r["row_pair"].cpu().numpy()
    assert np.array_equal(rt[p2r], np.arange(T * k) // k)
    assert np.array_equal(rp[p2r], np.arange(T * k))
    pad = np.ones(po[-1], bool)
    pad[p2r] = False
    assert (rt[: po[-1]][pad] == -1).all() and (rp[: po[-1]][pad] == -1).all()
    te = r["tile_expert"].cpu().numpy()
    for e in range(E):
        assert (te[po[e] // m_tile: po[e + 1] // m_tile] == e).all()
    act = r["active"].cpu().numpy()
    nz = np.nonzero(ref["counts"])[0]
    assert act[0] == nz.size and np.array_equal(act[1:1 + nz.size], nz)
    assert ops.device_status() == 0


def test_permute_flags_bad_ids_without_hanging(dev):
    ids = torch.tensor([[0, 1], [2, 9], [3, 3], [1, 0]], dtype=torch.int32, device=dev)
    assert ops.device_status(clear=True) == 0
    r = ops.moe_permute(ids, 4, 1)
    st = ops.device_status(clear=True)
    assert st & C.DEV_BAD_EXPERT_ID and st & C.DEV_DUPLICATE_ID
    p2r = r["pair_to_row"].cpu().numpy()
    assert p2r[3] == -1 and p2r[5] == -1 and (p2r[[0, 1, 2, 4, 6, 7]] >= 0).all()
    assert ops.device_status() == 0


# ------------------------------------------------------------------- GEMM ----
@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (3, 256, 512), (16, 384, 2048), (7, 128, 5120),
                                   (17, 128, 256), (128, 256, 512), (300, 512, 1024), (200, 384, 640),
                                   (513, 256, 2048)])
def test_gemm_parity(dev, M, N, K):
    """M <= 16: split-K GEMV; M > 16: tcgen05 block-scaled MMA (ragged M, N tiles of 128 and
    256, a K that ends in half a stage)."""
    g = torch.Generator().manual_seed(M * N + K)
    a = torch.randn(M, K, generator=g)
    b = torch.randn(N, K, generator=g) / K ** 0.5
    ac, asf, sa = O.quantize(a.numpy())
    bc, bsf, sb = O.quantize(b.numpy())
    ref = O.gemm(ac, asf, sa, bc, bsf, sb)
    t = lambda v: torch.from_numpy(np.ascontiguousarray(v)).to(dev)
    D = ops.nvfp4_gemm(t(ac), t(LY.to_mma(asf, K)), torch.tensor([sa], device=dev), t(bc),
                       t(LY.to_mma(bsf, K)), torch.tensor([sb], device=dev), out_dtype=torch.float32)
    torch.cuda.synchronize()
    d = D.cpu().numpy().astype(np.float64)
    # fp32 accumulation of exact block sums: relative to the sum of |terms|
    scale = np.abs(O.dequantize(ac, asf, sa)) @ np.abs(O.dequantize(bc, bsf, sb)).T
    assert (np.abs(d - ref) <= 1e-5 * scale + 1e-30).all()
    Db = ops.nvfp4_gemm(t(ac), t(LY.to_mma(asf, K)), torch.tensor([sa], device=dev), t(bc),
                        t(LY.to_mma(bsf, K)), torch.tensor([sb], device=dev), out_dtype=torch.bfloat16)
    G.check_out(G.bf16_bits(Db), ref)


def _mx_matrices(B, rows, K, seed):
    """MXFP4 matrices from the oracle's MX quantiser: rows of different magnitudes, a zero row
    and a zero block."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((B, rows, K)) * np.exp2(rng.integers(-5, 6, (B, rows, 1)))).astype(np.float32)
    x[0, 1] = 0.0
    x[-1, 2, 32:64] = 0.0
    mx = [O.mx_quantize(x[b]) for b in range(B)]
    return np.stack([m[0] for m in mx]), np.stack([m[1] for m in mx])


@pytest.mark.parametrize("B,rows,K", [(1, 3, 64), (3, 130, 256), (2, 256, 2048)])
def test_from_mxfp4_matches_oracle(dev, B, rows, K):
    """The exact NVFP4 form of MXFP4 matrices: codes unchanged, E4M3 block scales and the tensor
    scale bit-exact against the oracle's conversion (reading R11)."""
    codes, e8m0 = _mx_matrices(B, rows, K, seed=rows)
    c_d, sf_d, sc_d = ops.nvfp4_from_mxfp4(torch.from_numpy(codes).to(dev), torch.from_numpy(e8m0).to(dev))
    torch.cuda.synchronize()
    for b in range(B):
        _, sf_ref, sc_ref = O.mx_to_nvfp4(codes[b], e8m0[b])
        assert np.array_equal(LY.from_mma(sf_d[b].cpu().numpy(), rows, K), sf_ref)
        assert sc_d[b].item() == np.float32(sc_ref)
    assert np.array_equal(c_d.cpu().numpy(), codes)


def test_from_mxfp4_refuses_spans_without_an_exact_form(dev):
    y = np.ones((4, 64), np.float32)
    y[2, :32] = 2.0 ** -20  # 20 binades below the largest block
    c, e = O.mx_quantize(y)
    with pytest.raises(C.Nvfp4MoeError, match="18 binades"):
        ops.nvfp4_from_mxfp4(torch.from_numpy(c).to(dev), torch.from_numpy(e).to(dev))


@pytest.mark.parametrize("name", ["tiny", "decode_small"])
def test_from_nvfp4_gives_the_library_layout(dev, name):
    """Already-quantised NVFP4 experts (the oracle's codes, row-major E4M3 scales and tensor
    scales) prepared on the device (W13 interleave, MMA scales) equal, byte for byte, the
    layout the header defines, built on the host from the same arrays."""
    wl = {"tiny": W.WORKLOADS["tiny"], "decode_small": W.scaled(W.WORKLOADS["decode"], E=12, H=512, I=192)}[name]
    _, _, wg, wu, wd = G.layer_inputs(wl)
    up = [tuple(torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in w) for w in (wg, wu, wd)]
    got = ops.NVFP4Experts.from_nvfp4(*up)
    want = LY.experts_to_device_layout(wg, wu, wd)
    torch.cuda.synchronize()
    names = ("w13_codes", "w13_sf", "w13_scale", "w2_codes", "w2_sf", "w2_scale")
    for n, ref in zip(names, want):
        assert np.array_equal(getattr(got, n).cpu().numpy().reshape(ref.shape), ref), n
    assert ops.device_status() == 0


@pytest.mark.parametrize("B,rows,K", [(1, 5, 64), (3, 200, 192), (2, 256, 1024)])
def test_prep_weights_scale_layouts_round_trip(dev, B, rows, K):
    """Scales alone: row-major -> MMA equals the header's layout (padding rows untouched), and
    MMA -> row-major gives the input back."""
    rng = np.random.default_rng(rows)
    sf = rng.integers(0, 256, size=(B, rows * (K // 16)), dtype=np.uint8)
    mma = torch.zeros(B, LY.sf_mma_bytes(rows, K), dtype=torch.uint8, device=dev)
    _, mma = ops.nvfp4_prep_weights(None, torch.from_numpy(sf).to(dev), K, rows=rows, sf_out=mma)
    _, back = ops.nvfp4_prep_weights(None, mma, K, rows=rows, sf_layout=C.SF_MMA, sf_out_layout=C.SF_ROWMAJOR)
    torch.cuda.synchronize()
    for b in range(B):
        assert np.array_equal(mma[b].cpu().numpy(), LY.to_mma(sf[b].reshape(rows, K // 16), K))
    assert np.array_equal(back.cpu().numpy(), sf)


def test_prep_weights_reports_a_gather_past_the_input(dev):
    """A gather entry past the input rows is skipped and sets DEV_BAD_GATHER; the other rows
    are still written, a negative entry leaves its row as it was."""
    assert ops.device_status() == 0
    rows, K = 4, 64
    codes = torch.arange(rows * K // 2, dtype=torch.int32, device=dev).to(torch.uint8).reshape(rows, K // 2)
    sf = torch.arange(1, rows * K // 16 + 1, dtype=torch.uint8, device=dev)
    gather = torch.tensor([3, 9, -1, 0], dtype=torch.int32, device=dev)
    out = torch.full((4, K // 2), 0xAB, dtype=torch.uint8, device=dev)
    ops.nvfp4_prep_weights(codes, sf, K, row_gather=gather, out_rows=4, codes_out=out,
                           sf_out=torch.zeros(LY.sf_mma_bytes(4, K), dtype=torch.uint8, device=dev))
    assert ops.device_status(clear=True) == C.DEV_BAD_GATHER
    assert ops.device_status() == 0
    o = out.cpu()
    assert torch.equal(o[0], codes[3].cpu()) and torch.equal(o[3], codes[0].cpu())
    assert (o[1] == 0xAB).all() and (o[2] == 0xAB).all()


def test_from_mxfp4_rejects_a_gather_past_the_input(dev):
    codes, e8m0 = _mx_matrices(1, 4, 64, seed=3)
    gather = torch.tensor([0, 1, 7, -1], dtype=torch.int32, device=dev)  # row 7 does not exist
    with pytest.raises(C.Nvfp4MoeError, match="row_gather"):
        ops.nvfp4_from_mxfp4(torch.from_numpy(codes).to(dev), torch.from_numpy(e8m0).to(dev), gather, 4,
                             torch.zeros(1, 4, 32, dtype=torch.uint8, device=dev))


def test_bounded_wait_gives_up_and_reports_timeout(dev):
    """The bounded-wait path of the tcgen05 kernels, made to run out: a wait limited to a few
    polls on a barrier nothing arrives on gives up, sets the timeout bit of the device status
    word and returns; the context stays usable and the next call reports no fault."""
    ops.device_status(clear=True)
    assert ops.wait_selftest(4) == 0
    assert ops.device_status(clear=True) & C.DEV_TIMEOUT
    x = torch.randn(8, 64, device=dev)
    codes, sf, scale = ops.nvfp4_quantize(x)
    torch.cuda.synchronize()
    assert codes.shape == (8, 32) and float(scale.item()) > 0
    assert ops.device_status(clear=True) == 0


def test_mma_peak_probe_measures_a_plausible_ceiling(dev):
    """The FP4 MMA ceiling loop runs to completion (no bounded wait gives up) and gives a rate
    between a tenth of and twice the published dense FP4 figure (9 PFLOP/s)."""
    ops.device_status(clear=True)
    tf = ops.mma_peak_tflops(iters=4000, repeats=1)
    assert ops.device_status(clear=True) == 0
    assert 900.0 < tf < 18000.0, tf
