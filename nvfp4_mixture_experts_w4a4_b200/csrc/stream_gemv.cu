// Weight-only (W4A16) expert products for decode batches, streamed through shared memory.
//
// The weight-only layer (bf16 activations, NVFP4 weights; Qwen3.8-27B-nvfp4full-dflash2-NInfer
// card, "Limits") is bound by reading each touched expert's weights once.  A register-fed
// GEMV keeps too few bytes in flight per SM for HBM; here one warp per CTA streams the weight
// tiles with the copy engine (a 2-D tensor-map load of 128 rows x KSB bytes of codes and one
// bulk copy of their E4M3 scales per stage) into a ring of shared-memory stages, and eight
// warps compute from shared memory on the CUDA cores:
//   * a work item is one active expert's 128-row weight tile; its tokens (the expert's rows of
//     the unpadded permutation) are taken two at a time, their bf16 activation rows staged in
//     shared memory once per group of two;
//   * consumer warp w owns rows 16w..16w+15 of the tile; lane (rsel, cl) takes 16-byte chunk cl
//     (32 codes, two 16-element blocks) of rows 16w + 2p + rsel, p = 0..7; codes are widened
//     to f16 (exact); each token's activations are staged in f16 times a power of two that puts
//     their largest magnitude in [2^14, 2^15) (exact for every element within a factor 2^28 of it);
//     products are mixed f16 x f16 + fp32 fused multiply-adds (exact product, one fp32
//     rounding), the two block sums are fp32, each is multiplied by its E4M3 scale and the
//     power of two is taken back out of the row result; the 16 lanes of a row are summed with
//     a butterfly;
//   * gate/up: rows come as 16 gate rows then 16 up rows per 16-wide block of h; the epilogue
//     applies the tensor scales, h = silu(g) * u, rounded to bf16;
//   * down: the 128 rows are output features; each token's row is scaled by its routing
//     weight and the tensor scale and written to its pair's fp32 slot row.
// Every wait on a stage barrier is bounded; a timeout sets the device status word and the CTA
// stops waiting (the consumer warps still pass their named barriers together, doing no
// work, so none of them can be left at one; the producer lets its copies in flight land).
#include "ffn_gemv.cuh"
#include "gemv.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace nvfp4moe {
namespace {

using namespace sm100;

constexpr int kConsumers = 8;                       // consumer warps
constexpr int kThreadsS = (kConsumers + 1) * 32;    // + the producer warp
constexpr int kRows = 128;                          // weight rows per item
constexpr int kNT = 2;                              // tokens per group
constexpr uint32_t kStatusTimeout = 1u << 3;
constexpr int kSharedTok = kNT;                     // shared expert: tokens per work item (one group)

struct StreamParams {
  int K;            // reduction size (H for gate/up, I for down)
  int NW;           // weight rows per expert (2I or H)
  int KSB;          // code bytes per row per stage (divides K/2; multiple of 32)
  int stages;
  int n_mt;         // 128-row tiles per expert
  int H, I;
  const uint16_t* act;       // bf16 rows: x [T][H] (gate/up, by token) or h [P][I] (down, by row)
  const int32_t* offsets;    // [E+1]
  const int32_t* row_token;  // [P]
  const int32_t* row_pair;   // [P]
  const int32_t* active;     // [E+1]
  const uint8_t* w_sf;       // MMA layout per expert
  const float* w_scale;      // gate/up: [E][2]; down: [E]
  const float* topk_w;       // [P] by pair
  uint16_t* h_out;           // gate/up: bf16 [P][I]
  float* slots;              // down: fp32 [P][H] (shared expert: [T][H] by token, unweighted)
  uint32_t* status;
  int shared_T;              // > 0: the shared expert (one expert, tokens 0..T-1 in order, bf16 weights)
};

__device__ __forceinline__ void bar_consumers() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory"); }

// largest finite magnitude among eight bf16 values (0 if none)
__device__ __forceinline__ float finite_amax8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = fabsf(bf16_lo(w[i])), b = fabsf(bf16_hi(w[i]));
    if (a < __int_as_float(0x7F800000)) m = fmaxf(m, a);  // not inf, not NaN
    if (b < __int_as_float(0x7F800000)) m = fmaxf(m, b);
  }
  return m;
}

// p with amax * 2^p in [2^14, 2^15) (0 for amax 0), kept within [-126, 126] so that 2^p and
// 2^-p are normal fp32 values
__device__ __forceinline__ int act_shift(float amax) {
  if (!(amax > 0.0f)) return 0;
  const int e = int((__float_as_uint(amax) >> 23) & 0xFFu);
  return min(max(141 - max(e, 1), -126), 126);
}

// two bf16 values times the power of two sc, rounded to f16 (exact unless below the f16 normal range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float sc) {
  const __half2 h = __floats2half2_rn(bf16_lo(w) * sc, bf16_hi(w) * sc);
  return *reinterpret_cast<const uint32_t*>(&h);
}

struct GroupCtx {
  const uint8_t* sA;
  const uint8_t* sSF;
  const uint16_t* xs;
  float* sres;
  uint64_t* full;
  uint64_t* empty;
  volatile int* abort_flag;
  uint32_t* status;
  int S, KSB, K, kst, a_bytes, sf_bytes, warp, lane;
};

// The products of one token group with this warp's 16 rows over all K stages (NT tokens,
// a compile-time count so that no work or register is spent on absent tokens); the row
// results, times xd[t] (the inverse of token t's staging scale), land in sres[row][t].
// `it` counts stages consumed, `ok` turns false on a timeout.
template <int NT, bool WB>
__device__ __forceinline__ void group_products(const GroupCtx& c, const float (&xd)[kNT], uint32_t& it, bool& ok) {
  const int rsel = c.lane >> 4, cl = c.lane & 15;
  const bool chunk_on = cl * 16 < c.KSB;
  float acc[8][NT];
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[q][t] = 0.0f;
  for (int ks = 0; ks < c.kst; ++ks, ++it) {
    const int s = it % c.S;
    if (ok && *c.abort_flag) ok = false;
    if (ok && !mbar_wait(&c.full[s], (it / c.S) & 1)) {
      *c.abort_flag = 1;
      atomicOr(c.status, kStatusTimeout);
      ok = false;
    }
    if (WB && ok && chunk_on) {
      // bf16 weights: a 16-byte chunk is 8 weights, against this lane's 8 activations per token
      uint4 xv[NT];
      const int e0 = ks * (c.KSB / 2) + cl * 8;
#pragma unroll
      for (int t = 0; t < NT; ++t) xv[t] = *reinterpret_cast<const uint4*>(c.xs + t * c.K + e0);
      const uint8_t* a = c.sA + s * c.a_bytes;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int row = 16 * c.warp + 2 * q + rsel;
        const uint4 wv = *reinterpret_cast<const uint4*>(a + row * c.KSB + cl * 16);
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint32_t xw[4] = {xv[t].x, xv[t].y, xv[t].z, xv[t].w};
          float b = acc[q][t];
#pragma unroll
          for (int i = 0; i < 4; ++i) b = fma2_bf16_f32(ww[i], xw[i], b);
          acc[q][t] = b;
        }
      }
    }
    if (!WB && ok && chunk_on) {
      // this lane's 32 activation values of each token as f16 pairs (shared by its 8 rows)
      uint32_t xw[NT][16];
      const int e0 = ks * 2 * c.KSB + cl * 32;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const uint4* src = reinterpret_cast<const uint4*>(c.xs + t * c.K + e0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = src[i];
          xw[t][4 * i] = v.x;
          xw[t][4 * i + 1] = v.y;
          xw[t][4 * i + 2] = v.z;
          xw[t][4 * i + 3] = v.w;
        }
      }
      const uint8_t* a = c.sA + s * c.a_bytes;
      const uint8_t* sfs = c.sSF + s * c.sf_bytes;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int row = 16 * c.warp + 2 * q + rsel;
        const uint4 wv = *reinterpret_cast<const uint4*>(a + row * c.KSB + cl * 16);
        const uint32_t sfw = *reinterpret_cast<const uint16_t*>(sfs + (cl >> 1) * 512 + (row & 31) * 16 +
                                                                 ((row & 127) >> 5) * 4 + (cl & 1) * 2);
        uint32_t wf[16];
        decode_chunk(wv, wf);
        const float2 wsc = decode_sf2(sfw);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          float b0 = 0.0f, b1 = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) b0 = fma2_f16_f32(wf[i], xw[t][i], b0);
#pragma unroll
          for (int i = 8; i < 16; ++i) b1 = fma2_f16_f32(wf[i], xw[t][i], b1);
          acc[q][t] = __fmaf_rn(b1, wsc.y, __fmaf_rn(b0, wsc.x, acc[q][t]));
        }
      }
    }
    __syncwarp();
    if (ok && c.lane == 0) mbar_arrive(&c.empty[s]);
  }
  // sum the 16 chunk lanes of each row; lane cl == 0 parks the row's results
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float v = acc[q][t];
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (cl == 0) c.sres[(16 * c.warp + 2 * q + rsel) * kNT + t] = v * xd[t];
    }
}

// WB: bf16 weights (the shared expert), no block scales; otherwise NVFP4 codes + E4M3 scales.
template <int EPI, bool WB>
__global__ void __launch_bounds__(kThreadsS, 1) stream_gemv_kernel(const __grid_constant__ CUtensorMap tmW, StreamParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_shared_1024(smem_raw);
  const int S = p.stages, KSB = p.KSB, K = p.K;
  const int a_bytes = kRows * KSB, sf_bytes = WB ? 0 : 16 * KSB;  // KSB / 32 scale atoms of 512 bytes
  uint8_t* sA = smem;
  uint8_t* sSF = sA + S * a_bytes;
  uint16_t* xs = reinterpret_cast<uint16_t*>(sSF + S * sf_bytes);  // [kNT][K] bf16
  float* sres = reinterpret_cast<float*>(xs + kNT * K);             // [kRows][kNT]
  float* sred = sres + kRows * kNT;                                 // [kConsumers][kNT] amax partials
  uint64_t* full = reinterpret_cast<uint64_t*>(sred + kConsumers * kNT);
  uint64_t* empty = full + S;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + S);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kConsumers && lane == 0) prefetch_tensormap(&tmW);
  __syncthreads();
  griddep_wait();  // the routing step's counts and, for down, the gate/up output

  // the shared expert's items are (weight tile, one token group): every SM takes part, and no item
  // streams its weight tile twice
  const bool shared = p.shared_T > 0;
  const int n_items = (shared ? (p.shared_T + kSharedTok - 1) / kSharedTok : p.active[0]) * p.n_mt;
  const int kst = (WB ? 2 * K : K / 2) / KSB;  // stages per pass over K
  auto abort_now = [&]() {
    *abort_flag = 1;
    atomicOr(p.status, kStatusTimeout);
  };

  if (warp == kConsumers) {
    // ------------------------------------------------------------- producer ----
    if (elect_one()) {
      uint32_t it = 0;
      for (int item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x) {
        const int e = shared ? 0 : p.active[1 + item / p.n_mt], mt = item % p.n_mt;
        const int t0 = (item / p.n_mt) * kSharedTok;
        const int n_e = shared ? min(kSharedTok, p.shared_T - t0) : p.offsets[e + 1] - p.offsets[e];
        const int64_t row0 = int64_t(e) * p.NW + int64_t(mt) * kRows;
        const uint8_t* sf = WB ? nullptr : p.w_sf + row0 * (K / 16);
        for (int g = 0; g < n_e && !*abort_flag; g += kNT)
          for (int ks = 0; ks < kst; ++ks, ++it) {
            const int s = it % S;
            if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1)) {
              abort_now();
              break;
            }
            mbar_arrive_expect_tx(&full[s], a_bytes + sf_bytes);
            tma_load_2d(sA + s * a_bytes, &tmW, ks * KSB, static_cast<int32_t>(row0), &full[s]);
            if (!WB) bulk_load(sSF + s * sf_bytes, sf + int64_t(ks) * sf_bytes, sf_bytes, &full[s]);
          }
      }
      if (*abort_flag)  // let the copies in flight land before the CTA exits
        for (uint32_t back = 0; back < uint32_t(S) && back < it; ++back) {
          const uint32_t jj = it - 1 - back;
          mbar_wait(&full[jj % S], (jj / S) & 1, 1u << 16);
        }
    }
    return;
  }

  // ------------------------------------------------------------- consumers ----
  const GroupCtx g_args{sA, sSF, xs, sres, full, empty, abort_flag, p.status, S, KSB, K, kst, a_bytes, sf_bytes, warp,
                        lane};
  uint32_t it = 0;
  bool ok = true;  // false once a wait timed out (here or in another warp): no more waits
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int e = shared ? 0 : p.active[1 + item / p.n_mt], mt = item % p.n_mt;
    const int r0 = shared ? (item / p.n_mt) * kSharedTok : p.offsets[e];
    const int n_e = shared ? min(kSharedTok, p.shared_T - r0) : p.offsets[e + 1] - r0;
    for (int g = 0; g < n_e; g += kNT) {
      const int nt = min(kNT, n_e - g);
      // stage the group's activation rows (zeros past nt)
      const int vec_per_row = K / 8;  // 16-byte vectors of one bf16 row
      float lmax[kNT];
#pragma unroll
      for (int t = 0; t < kNT; ++t) lmax[t] = 0.0f;
      for (int v = threadIdx.x; v < kNT * vec_per_row; v += kConsumers * 32) {
        const int t = v / vec_per_row, c = v - t * vec_per_row;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (t < nt) {
          const int64_t src_row = EPI == 0 && !shared ? int64_t(p.row_token[r0 + g + t]) : int64_t(r0 + g + t);
          val = __ldg(reinterpret_cast<const uint4*>(p.act + src_row * K) + c);
        }
        reinterpret_cast<uint4*>(xs + t * K)[c] = val;
        if (!WB) {
          const float am = finite_amax8(val);
#pragma unroll
          for (int u = 0; u < kNT; ++u)  // (unrolled: no local-memory array)
            if (t == u) lmax[u] = fmaxf(lmax[u], am);
        }
      }
      // NVFP4 weights: each token's row becomes f16 times 2^p_t, p_t putting its largest finite
      // magnitude in [2^14, 2^15); the row results are scaled back by 2^-p_t
      float xd[kNT];
#pragma unroll
      for (int t = 0; t < kNT; ++t) xd[t] = 1.0f;
      if (!WB) {
#pragma unroll
        for (int t = 0; t < kNT; ++t) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) lmax[t] = fmaxf(lmax[t], __shfl_xor_sync(0xffffffffu, lmax[t], o));
          if (lane == 0) sred[warp * kNT + t] = lmax[t];
        }
        bar_consumers();
        float xsc[kNT];
#pragma unroll
        for (int t = 0; t < kNT; ++t) {
          float m = sred[t];
#pragma unroll
          for (int w = 1; w < kConsumers; ++w) m = fmaxf(m, sred[w * kNT + t]);
          const int sh = act_shift(m);
          xsc[t] = __uint_as_float(uint32_t(127 + sh) << 23);
          xd[t] = __uint_as_float(uint32_t(127 - sh) << 23);
        }
        for (int v = threadIdx.x; v < kNT * vec_per_row; v += kConsumers * 32) {
          const int t = v / vec_per_row, c = v - t * vec_per_row;
          uint4* ptr = reinterpret_cast<uint4*>(xs + t * K) + c;
          float sc = xsc[0];
#pragma unroll
          for (int u = 1; u < kNT; ++u)
            if (t == u) sc = xsc[u];
          const uint4 raw = *ptr;
          *ptr = make_uint4(bf16x2_to_f16x2(raw.x, sc), bf16x2_to_f16x2(raw.y, sc), bf16x2_to_f16x2(raw.z, sc),
                            bf16x2_to_f16x2(raw.w, sc));
        }
      }
      bar_consumers();
      if (nt == 1)
        group_products<1, WB>(g_args, xd, it, ok);
      else
        group_products<2, WB>(g_args, xd, it, ok);
      bar_consumers();
      const int l = lane & 15, tt = lane >> 4;
      if (!ok) continue;  // (the next group's barriers are still passed by every warp)
      if (EPI == 0) {
        // warps 0..3: one 16-wide block of h each (gate rows 32w.., up rows 32w+16..)
        if (warp < 4) {
          const float sg = WB ? 1.0f : p.w_scale[2 * e], su = WB ? 1.0f : p.w_scale[2 * e + 1];
          const int col = (mt * 4 + warp) * 16 + l;
          for (int t = tt; t < nt; t += 2) {
            const float gv = sres[(32 * warp + l) * kNT + t] * sg;
            const float uv = sres[(32 * warp + 16 + l) * kNT + t] * su;
            const float h = gv / (1.0f + expf(-gv)) * uv;
            const __nv_bfloat16 hb = __float2bfloat16_rn(h);
            p.h_out[int64_t(r0 + g + t) * p.I + col] = *reinterpret_cast<const uint16_t*>(&hb);
          }
        }
      } else {
        // each warp writes its 16 output features of every token to the token's slot row
        const float sw = WB ? 1.0f : p.w_scale[e];
        const int n = mt * kRows + 16 * warp + l;
        for (int t = tt; t < nt; t += 2) {
          if (shared) {  // the shared expert's row of token g + t, unweighted
            p.slots[int64_t(r0 + g + t) * p.H + n] = sres[(16 * warp + l) * kNT + t];
            continue;
          }
          const int32_t pair = p.row_pair[r0 + g + t];
          p.slots[int64_t(pair) * p.H + n] = sres[(16 * warp + l) * kNT + t] * sw * p.topk_w[pair];
        }
      }
    }
  }
}

}  // namespace

nvfp4moe_status launch_stream_gemv_a16(int epi, const StreamA16Args& a, int64_t max_active, cudaStream_t s) {
  uint32_t* status = device_status_ptr();
  if (!status) return fail(NVFP4MOE_CUDA_ERROR, "device status word unavailable");
  const bool wb = a.wbf16 != 0;
  StreamParams p{};
  p.K = epi == 0 ? a.H : a.I;
  p.NW = epi == 0 ? 2 * a.I : a.H;
  const int row_bytes = wb ? 2 * p.K : p.K / 2;  // weight bytes per row
  p.KSB = row_bytes % 256 == 0 ? 256 : row_bytes % 128 == 0 ? 128 : row_bytes % 64 == 0 ? 64 : 32;
  if (row_bytes % p.KSB != 0 || p.NW % kRows != 0)
    return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "stream GEMV: K=%d, rows=%d", p.K, p.NW);
  p.n_mt = p.NW / kRows;
  p.H = a.H;
  p.I = a.I;
  p.act = a.act;
  p.offsets = a.offsets;
  p.row_token = a.row_token;
  p.row_pair = a.row_pair;
  p.active = a.active;
  p.w_sf = a.w_sf;
  p.w_scale = a.w_scale;
  p.topk_w = a.topk_w;
  p.h_out = a.h_out;
  p.slots = a.slots;
  p.status = status;
  p.shared_T = a.shared_T;
  const int stage_bytes = kRows * p.KSB + (wb ? 0 : 16 * p.KSB);
  const int fixed = 1024 + kNT * p.K * 2 + kRows * kNT * 4 + kConsumers * kNT * 4 + 64;
  const int budget = 227 * 1024;
  int stages = (budget - fixed - 16 * 8) / stage_bytes;
  if (stages > 6) stages = 6;
  if (stages < 2) return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "stream GEMV: K=%d leaves no room", p.K);
  p.stages = stages;
  const size_t smem = size_t(fixed) + size_t(stages) * (stage_bytes + 16);

  // weights as [E*NW][row_bytes] bytes, box KSB bytes x 128 rows, no swizzle
  auto fn = tensor_map_encoder();
  if (!fn) return fail(NVFP4MOE_CUDA_ERROR, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap map;
  const int64_t rows = int64_t(a.E) * p.NW;
  const cuuint64_t dims[2] = {cuuint64_t(row_bytes), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(row_bytes)};
  const cuuint32_t box[2] = {cuuint32_t(p.KSB), cuuint32_t(kRows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.w_codes), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4MOE_CUDA_ERROR, "cuTensorMapEncodeTiled (stream GEMV) failed (%d)", int(r));

  const int64_t items =
      (a.shared_T > 0 ? (int64_t(a.shared_T) + kSharedTok - 1) / kSharedTok : max_active) * p.n_mt;
  const int grid = static_cast<int>(items < num_sms() ? (items > 0 ? items : 1) : num_sms());
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err == cudaSuccess) err = launch_dependent(kern, dim3(grid), dim3(kThreadsS), smem, s, map, p);
    return err;
  };
  const cudaError_t e = epi == 0 ? (wb ? go(stream_gemv_kernel<0, true>) : go(stream_gemv_kernel<0, false>))
                                 : (wb ? go(stream_gemv_kernel<1, true>) : go(stream_gemv_kernel<1, false>));
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "stream GEMV: %s", cudaGetErrorString(e));
  return check_launch("stream GEMV");
}

}  // namespace nvfp4moe
