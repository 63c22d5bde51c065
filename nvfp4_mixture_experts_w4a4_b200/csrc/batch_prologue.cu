// Prologue of the routed layer for batches above the cluster prologue's 64 tokens: router
// top-k, the expert permutation and the activation quantisation, writing exactly what
// moe_route, moe_permute and nvfp4_quantize (plus the copy into expert order) write, in three
// launches over slices of up to 32 tokens (sized to give about two CTAs per SM):
//   1. route_hist_kernel   one CTA per slice: warp_topk per token (as moe_route), the slice's
//                          expert histogram, and the amax of its x rows (dynamic scale);
//   2. col_scan_kernel     per expert, the exclusive prefix of the slice histograms (in place:
//                          the histogram becomes each slice's first rank) and the count;
//   3. place_quant_kernel  one CTA per slice: expert offsets and padded offsets from one block
//                          scan of the counts (CTA 0 also writes them and the active list),
//                          the x scale from the partial maxima; each pair's row = padded offset of its expert +
//                          the slice's first rank + the number of earlier tokens of the slice
//                          with that expert (a 32-bit token mask per expert and a popcount),
//                          so rows of an expert follow token order, the stable order of
//                          moe_permute; then each 16-element block of the slice's x rows is
//                          quantised once and written to its k rows (or, GEMV layout, to the
//                          token's row); padding rows and the tile map, split over the CTAs.
// Kernels 2 and 3 are launched as programmatic dependents and wait for their predecessor.
#include "topk.cuh"

namespace nvfp4moe {
namespace {

constexpr int kSlice = 32;      // tokens per slice at most (token masks are 32-bit)
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int MAX_E = 1024;
constexpr int MAX_K = 32;

struct BatchArgs {
  const __nv_bfloat16* x;   // [T][H]
  const float* logits;      // [T][E]
  int T, H, E, k;
  int m_tile_log2;
  int dynamic;              // 1: x scale = amax / 2688, written to *x_scale; 0: read *x_scale
  float* x_scale;
  int32_t* ids;             // [T][k]
  float* w;                 // [T][k]
  int32_t *counts, *offsets, *padded_offsets, *pair_to_row, *row_token, *row_pair, *tile_expert, *active;
  float* zero_f32;          // nullable [E]
  int expert_order;         // 1: x rows go to the padded expert-order rows; 0: token-major
  uint8_t* x_codes;         // nullable: x is not quantised (weight-only layer)
  uint8_t* x_sf;            // MMA layout
  int32_t* hist;            // [slices][E] histogram, then each slice's first rank per expert
  float* partials;          // [slices] amax of each slice's x rows
  float* zero_rows;         // nullable [T][H] fp32: each slice's rows are zeroed
  int slices;
  int slice;                // tokens per slice
};

template <int PER_LANE>
__global__ void __launch_bounds__(kThreads) route_hist_kernel(BatchArgs a) {
  __shared__ int32_t s_hist[MAX_E];
  __shared__ float s_red[kWarps];
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = blockIdx.x * a.slice;
  const int nt = min(a.slice, a.T - t0);
  for (int e = threadIdx.x; e < a.E; e += kThreads) s_hist[e] = 0;
  __syncthreads();
  for (int tl = warp; tl < nt; tl += kWarps) {
    const int t = t0 + tl;
    int id;
    float wt;
    warp_topk<PER_LANE>(a.logits + int64_t(t) * a.E, a.E, a.k, &id, &wt);
    if (lane < a.k) {
      a.ids[int64_t(t) * a.k + lane] = id;
      a.w[int64_t(t) * a.k + lane] = wt;
      atomicAdd(&s_hist[id], 1);
    }
  }
  if (a.dynamic) {
    float m = 0.0f;
    const int64_t chunks = int64_t(nt) * a.H / 8;
    const uint4* base = reinterpret_cast<const uint4*>(a.x + int64_t(t0) * a.H);
    for (int64_t i0 = threadIdx.x; i0 < chunks; i0 += 4 * kThreads) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t i = i0 + int64_t(j) * kThreads;
        u[j] = i < chunks ? __ldg(base + i) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t q[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
        for (int h = 0; h < 4; ++h)
          m = fmaxf(m, fmaxf(fabsf(__uint_as_float(q[h] << 16)), fabsf(__uint_as_float(q[h] & 0xFFFF0000u))));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_red[warp] = m;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += kThreads) a.hist[int64_t(blockIdx.x) * a.E + e] = s_hist[e];
  if (a.dynamic && threadIdx.x == 0) {
    float r = 0.0f;
    for (int i = 0; i < kWarps; ++i) r = fmaxf(r, s_red[i]);
    a.partials[blockIdx.x] = r;
  }
}

// Column scan: CTA b owns experts 32b .. 32b+31 (the lanes) and splits the slices into 32
// ranges (the warps); the slice histograms become each slice's first rank per expert, and
// the expert totals are the counts.
__global__ void __launch_bounds__(1024) col_scan_kernel(BatchArgs a) {
  __shared__ int32_t s_sum[32][33];
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, part = threadIdx.x >> 5;
  const int E = a.E;
  const int e = blockIdx.x * 32 + lane;
  const int64_t c_lo = int64_t(a.slices) * part / 32, c_hi = int64_t(a.slices) * (part + 1) / 32;
  int run = 0;
  if (e < E) {
    int64_t c = c_lo;
    for (; c + 8 <= c_hi; c += 8) {
      int h[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) h[j] = a.hist[(c + j) * E + e];
#pragma unroll
      for (int j = 0; j < 8; ++j) run += h[j];
    }
    for (; c < c_hi; ++c) run += a.hist[c * E + e];
  }
  s_sum[part][lane] = run;
  __syncthreads();
  if (e < E) {
    int r = 0;
    for (int q = 0; q < part; ++q) r += s_sum[q][lane];
    int64_t c = c_lo;
    for (; c + 8 <= c_hi; c += 8) {
      int h[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) h[j] = a.hist[(c + j) * E + e];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        a.hist[(c + j) * E + e] = r;
        r += h[j];
      }
    }
    for (; c < c_hi; ++c) {
      const int h = a.hist[c * E + e];
      a.hist[c * E + e] = r;
      r += h;
    }
    if (part == 31) a.counts[e] = r;
  }
}

__global__ void __launch_bounds__(kThreads) place_quant_kernel(BatchArgs a) {
  __shared__ uint32_t s_mask[MAX_E];
  __shared__ int32_t s_start[MAX_E];
  __shared__ int32_t s_poff[MAX_E + 1];
  __shared__ int32_t s_cnt[MAX_E];
  __shared__ int32_t s_id[kSlice * MAX_K];
  __shared__ int32_t s_row[kSlice * MAX_K];
  __shared__ unsigned long long s_w64[kWarps];
  __shared__ int32_t s_w32[kWarps];
  __shared__ float s_red[kWarps];
  griddep_wait();
  griddep_launch_dependents();
  const int E = a.E, k = a.k, H = a.H;
  const int c = blockIdx.x;
  const int t0 = c * a.slice;
  const int nt = min(a.slice, a.T - t0);
  const int np = nt * k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  static_assert(MAX_E == 2 * kThreads, "two experts per thread");
  // counts and this slice's first ranks of experts 2t, 2t+1; the slice's ids; partial maxima
  int cnt[2], first[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int e = 2 * int(threadIdx.x) + i;
    cnt[i] = e < E ? a.counts[e] : 0;
    first[i] = e < E ? a.hist[int64_t(c) * E + e] : 0;
  }
  for (int pl = threadIdx.x; pl < np; pl += kThreads) s_id[pl] = a.ids[int64_t(t0) * k + pl];
  float m = 0.0f;
  if (a.dynamic)
    for (int i = threadIdx.x; i < a.slices; i += kThreads) m = fmaxf(m, a.partials[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // expert offsets, padded offsets and active slots: one block scan of the counts
  const int mt = 1 << a.m_tile_log2;
  unsigned long long v[2];
  int fl[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int pad = (cnt[i] + mt - 1) >> a.m_tile_log2 << a.m_tile_log2;
    v[i] = (static_cast<unsigned long long>(pad) << 32) | static_cast<unsigned>(cnt[i]);
    fl[i] = cnt[i] > 0;
  }
  unsigned long long incl = v[0] + v[1];
  int fincl = fl[0] + fl[1];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
    const int z = __shfl_up_sync(0xffffffffu, fincl, o);
    if (lane >= o) {
      incl += y;
      fincl += z;
    }
  }
  if (lane == 31) {
    s_w64[warp] = incl;
    s_w32[warp] = fincl;
  }
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  unsigned long long before = incl - v[0] - v[1];
  int fbefore = fincl - fl[0] - fl[1];
  for (int w = 0; w < warp; ++w) {
    before += s_w64[w];
    fbefore += s_w32[w];
  }
  unsigned long long total = 0;
  int ftotal = 0;
  float mx = 0.0f;
  for (int w = 0; w < kWarps; ++w) {
    total += s_w64[w];
    ftotal += s_w32[w];
    mx = fmaxf(mx, s_red[w]);
  }
  // (no x codes: the weight-only layer keeps x in bf16 and has no x scale)
  const float s_t = a.dynamic ? __fdiv_rn(mx, 2688.0f) : (a.x_codes ? *a.x_scale : 0.0f);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int e = 2 * int(threadIdx.x) + i;
    if (e < E) {
      const int po = static_cast<int>(before >> 32);
      s_poff[e] = po;
      s_cnt[e] = cnt[i];
      s_start[e] = po + first[i];
      s_mask[e] = 0u;
      if (c == 0) {
        a.offsets[e] = static_cast<int32_t>(before & 0xFFFFFFFFu);
        a.padded_offsets[e] = po;
        if (fl[i]) a.active[1 + fbefore] = e;
        if (a.zero_f32) a.zero_f32[e] = 0.0f;
      }
    }
    before += v[i];
    fbefore += fl[i];
  }
  if (threadIdx.x == 0) {
    s_poff[E] = static_cast<int>(total >> 32);
    if (c == 0) {
      a.offsets[E] = static_cast<int32_t>(total & 0xFFFFFFFFu);
      a.padded_offsets[E] = static_cast<int32_t>(total >> 32);
      a.active[0] = ftotal;
      if (a.dynamic) *a.x_scale = s_t;
    }
  }
  __syncthreads();
  for (int pl = threadIdx.x; pl < np; pl += kThreads) atomicOr(&s_mask[s_id[pl]], 1u << (pl / k));
  __syncthreads();
  for (int pl = threadIdx.x; pl < np; pl += kThreads) {
    const int e = s_id[pl];
    const int tl = pl / k;
    const int row = s_start[e] + __popc(s_mask[e] & ((1u << tl) - 1u));
    s_row[pl] = row;
    const int64_t p = int64_t(t0) * k + pl;
    a.pair_to_row[p] = row;
    a.row_token[row] = t0 + tl;
    a.row_pair[row] = static_cast<int32_t>(p);
  }
  __syncthreads();

  // quantise each 16-element block of the slice's x rows once; write it to its row(s)
  const int nb = H / 16;
  const int64_t rb = H / 2;
  const int n_items = a.x_codes ? nt * nb : 0;
  for (int item0 = threadIdx.x; item0 < n_items; item0 += 2 * kThreads) {
   uint4 uu[2][2];
#pragma unroll
   for (int h2 = 0; h2 < 2; ++h2) {
     const int item = item0 + h2 * kThreads;
     if (item < n_items) {
       const int tl = item / nb, b = item - tl * nb;
       const uint4* src = reinterpret_cast<const uint4*>(a.x + int64_t(t0 + tl) * H + b * 16);
       uu[h2][0] = __ldg(src);
       uu[h2][1] = __ldg(src + 1);
     }
   }
#pragma unroll
   for (int h2 = 0; h2 < 2; ++h2) {
    const int item = item0 + h2 * kThreads;
    if (item >= n_items) break;
    const int tl = item / nb, b = item - tl * nb;
    const uint4 u0 = uu[h2][0], u1 = uu[h2][1];
    const uint32_t q[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    float v[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[2 * j] = __uint_as_float(q[j] << 16);
      v[2 * j + 1] = __uint_as_float(q[j] & 0xFFFF0000u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    float inv;
    const uint32_t sf = block_scale(amax, s_t, &inv);
    const uint2 code = encode_block16(v, inv);
    const int n_dst = a.expert_order ? k : 1;
    for (int d = 0; d < n_dst; ++d) {
      const int64_t row = a.expert_order ? s_row[tl * k + d] : t0 + tl;
      *reinterpret_cast<uint2*>(a.x_codes + row * rb + b * 8) = code;
      a.x_sf[sf_mma_offset(row, b, H)] = static_cast<uint8_t>(sf);
    }
   }
  }

  // the accumulating combine's output rows of this slice start at zero
  if (a.zero_rows) {
    float4* z = reinterpret_cast<float4*>(a.zero_rows + int64_t(t0) * H);
    for (int64_t i = threadIdx.x; i < int64_t(nt) * H / 4; i += kThreads) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // padding rows and the tile -> expert map for this CTA's share of the padded rows: row r
  // belongs to the last expert whose padded offset is <= r
  const int64_t rows = s_poff[E];
  const int64_t r_lo = rows * c / gridDim.x, r_hi = rows * (c + 1) / gridDim.x;
  const int mmask = (1 << a.m_tile_log2) - 1;
  for (int64_t r = r_lo + threadIdx.x; r < r_hi; r += kThreads) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_poff[mid] <= r) lo = mid; else hi = mid - 1;
    }
    if (r - s_poff[lo] >= s_cnt[lo]) {
      a.row_token[r] = -1;
      a.row_pair[r] = -1;
    }
    if ((r & mmask) == 0) a.tile_expert[r >> a.m_tile_log2] = lo;
  }
}

}  // namespace

bool batch_prologue_fits(int T, int E, int k) { return T >= 1 && E >= 1 && E <= MAX_E && k >= 1 && k <= MAX_K; }

// tokens per slice: about two slices per SM, at most kSlice
int slice_tokens(int T) {
  const int target = 2 * num_sms();
  const int per = (T + target - 1) / target;
  return per < 1 ? 1 : (per > kSlice ? kSlice : per);
}

int64_t batch_prologue_scratch_bytes(int T, int E) {
  const int64_t slices = (int64_t(T) + slice_tokens(T) - 1) / slice_tokens(T);
  return (slices * E * 4 + 255) / 256 * 256 + (slices * 4 + 255) / 256 * 256;
}

nvfp4moe_status launch_batch_prologue(const void* x, const float* logits, int T, int H, int E, int k, int m_tile,
                                      int dynamic, float* x_scale, int32_t* ids, float* w, int32_t* counts,
                                      int32_t* offsets, int32_t* padded_offsets, int32_t* pair_to_row,
                                      int32_t* row_token, int32_t* row_pair, int32_t* tile_expert, int32_t* active,
                                      float* zero_f32, int expert_order, uint8_t* x_codes, uint8_t* x_sf,
                                      void* scratch, float* zero_rows, void* const* stage_events, cudaStream_t s) {
  NVFP4_REQUIRE(batch_prologue_fits(T, E, k), NVFP4MOE_UNSUPPORTED_SHAPE, "batch prologue: T=%d E=%d k=%d out of range",
                T, E, k);
  int lg = 0;
  while ((1 << lg) < m_tile) ++lg;
  NVFP4_REQUIRE((1 << lg) == m_tile, NVFP4MOE_INVALID_ARG, "batch prologue: m_tile %d is not a power of two", m_tile);
  BatchArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.logits = logits;
  a.T = T; a.H = H; a.E = E; a.k = k; a.m_tile_log2 = lg;
  a.dynamic = dynamic; a.x_scale = x_scale;
  a.ids = ids; a.w = w;
  a.counts = counts; a.offsets = offsets; a.padded_offsets = padded_offsets; a.pair_to_row = pair_to_row;
  a.row_token = row_token; a.row_pair = row_pair; a.tile_expert = tile_expert; a.active = active;
  a.zero_f32 = zero_f32;
  a.expert_order = expert_order;
  a.x_codes = x_codes; a.x_sf = x_sf;
  a.zero_rows = zero_rows;
  a.slice = slice_tokens(T);
  a.slices = (T + a.slice - 1) / a.slice;
  a.hist = static_cast<int32_t*>(scratch);
  a.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + (int64_t(a.slices) * E * 4 + 255) / 256 * 256);
  auto mark = [&](int i) -> cudaError_t { return stage_events ? record_mark(stage_events[i], s) : cudaSuccess; };

  const int per = (E + 31) / 32;
  const dim3 grid(static_cast<unsigned>(a.slices));
  if (per <= 1)
    route_hist_kernel<1><<<grid, kThreads, 0, s>>>(a);
  else if (per <= 4)
    route_hist_kernel<4><<<grid, kThreads, 0, s>>>(a);
  else if (per <= 8)
    route_hist_kernel<8><<<grid, kThreads, 0, s>>>(a);
  else if (per <= 16)
    route_hist_kernel<16><<<grid, kThreads, 0, s>>>(a);
  else
    route_hist_kernel<32><<<grid, kThreads, 0, s>>>(a);
  nvfp4moe_status st = check_launch("batch prologue (route)");
  if (st != NVFP4MOE_OK) return st;
  cudaError_t e = mark(1);
  if (e == cudaSuccess) e = launch_dependent(col_scan_kernel, dim3(static_cast<unsigned>((E + 31) / 32)), dim3(1024), 0, s, a);
  if (e == cudaSuccess) e = mark(2);
  if (e == cudaSuccess) e = launch_dependent(place_quant_kernel, grid, dim3(kThreads), 0, s, a);
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "batch prologue: %s", cudaGetErrorString(e));
  return check_launch("batch prologue");
}

}  // namespace nvfp4moe
