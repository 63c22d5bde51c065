// Small-batch prologue of the routed layer: router top-k, the expert permutation and the
// activation quantisation (dynamic or given tensor scale) in ONE launch of one 8-CTA thread
// block cluster, writing exactly what moe_route, moe_permute and nvfp4_quantize (plus the
// copy into expert order) write.
//
// For decode-sized batches those steps move only kilobytes, so their cost is latency: a
// chain of dependent memory round trips and launches.  The cluster keeps the chain short:
//   1. CTA c routes the tokens t = c, c + 8, ... (one warp per token, warp_topk as moe_route)
//      and takes the amax of its 1/8 of x; each routing lane stores its expert id, and each
//      CTA its partial amax, into the shared memory of all eight CTAs (distributed shared
//      memory), then the cluster barrier makes every CTA hold all T*k ids and all maxima.
//   2. Every CTA then derives the whole permutation locally: a 64-bit token mask per expert
//      (T <= 64) gives each pair's rank inside its expert in one popcount, counts are the
//      masks' popcounts, and one block scan gives the offsets.  Because pairs are ordered
//      by token and a token names an expert at most once, rank = number of earlier tokens
//      with the same expert: the stable order of moe_permute.
//   3. The cluster's 2048 threads split the global writes (permutation arrays, pad rows,
//      tile map) and the quantisation: each thread quantises 16-element blocks of x once and
//      writes the codes to the token's row (GEMV layout) or to its k expert rows.
#include "topk.cuh"

namespace nvfp4moe {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int MAX_T = kCluster * kWarps;  // one routing warp per token
constexpr int MAX_P = MAX_T * 32;         // top_k <= 32
constexpr int MAX_E = 1024;
static_assert(MAX_E == 4 * kThreads, "the expert scan gives each thread four experts");
static_assert(MAX_T <= 64, "token masks are 64-bit");

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// 32-bit store into CTA `rank`'s copy of the shared-memory word at local address `addr`
__device__ __forceinline__ void st_cluster(uint32_t addr, uint32_t rank, uint32_t v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(remote), "r"(v) : "memory");
}

struct PrologueArgs {
  const __nv_bfloat16* x;   // [T][H]
  const float* logits;      // [T][E]
  int T, H, E, k;
  int m_tile_log2;          // row padding of each expert: 1 << m_tile_log2
  int dynamic;              // 1: x scale = amax / 2688 written to *x_scale; 0: read *x_scale
  float* x_scale;
  int32_t* ids;             // [T][k]
  float* w;                 // [T][k]
  int32_t *counts, *offsets, *padded_offsets, *pair_to_row, *row_token, *row_pair, *tile_expert, *active;
  float* zero_f32;          // nullable [E]
  int expert_order;         // 1: x rows go to the padded expert-order rows; 0: token-major
  uint8_t* x_codes;         // nullable: x is not quantised (weight-only layer)
  uint8_t* x_sf;            // MMA layout
  int4* list;               // nullable: the fused grouped GEMM's work list (one chunk per expert)
  int* done;                //   and its per-expert counters, zeroed here
  int wt_gateup, wt_down;   // weight tiles per expert of each GEMM
};

template <int PER_LANE>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1) prologue_kernel(PrologueArgs a) {
  __shared__ int32_t s_ids[MAX_P];
  __shared__ int32_t s_row[MAX_P];
  __shared__ unsigned long long s_mask[MAX_E];
  __shared__ int32_t s_cnt[MAX_E];
  __shared__ int32_t s_off[MAX_E + 1], s_poff[MAX_E + 1], s_aoff[MAX_E + 1];
  __shared__ int32_t s_act[MAX_E];  // active slot -> expert
  __shared__ float s_part[kCluster];
  __shared__ unsigned long long s_wsum[kWarps];
  __shared__ float s_red[kWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = static_cast<int>(cluster_rank());
  const int T = a.T, H = a.H, E = a.E, k = a.k, P = T * k;
  const int gi = c * kThreads + tid;
  constexpr int kAll = kCluster * kThreads;

  griddep_launch_dependents();  // the grouped GEMM may take the other SMs and set itself up
  // every CTA must have started before any writes into its shared memory
  cluster_arrive_relaxed();
  for (int e = tid; e < E; e += kThreads) s_mask[e] = 0ull;

  // ---- 1. route this CTA's tokens; partial amax of x -------------------------------------
  // The first x chunks are requested before the top-k so that both loads are in flight at once.
  const int64_t chunks = a.dynamic ? int64_t(T) * H / 8 : 0;  // 16-byte chunks of x
  const int64_t per = (chunks + kCluster - 1) / kCluster;
  const int64_t lo = c * per, hi = min(chunks, lo + per);
  const uint4* base = reinterpret_cast<const uint4*>(a.x);
  uint4 first[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int64_t i = lo + tid + int64_t(j) * kThreads;
    first[j] = i < hi ? __ldg(base + i) : make_uint4(0u, 0u, 0u, 0u);
  }
  const int t = c + kCluster * warp;
  int my_id = 0;
  float my_w = 0.0f;
  if (t < T) warp_topk<PER_LANE>(a.logits + int64_t(t) * E, E, k, &my_id, &my_w);
  float m = 0.0f;
  if (a.dynamic) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t q[4] = {first[j].x, first[j].y, first[j].z, first[j].w};
#pragma unroll
      for (int h = 0; h < 4; ++h)
        m = fmaxf(m, fmaxf(fabsf(__uint_as_float(q[h] << 16)), fabsf(__uint_as_float(q[h] & 0xFFFF0000u))));
    }
    for (int64_t i0 = lo + tid + 2 * kThreads; i0 < hi; i0 += 4 * kThreads) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t i = i0 + int64_t(j) * kThreads;
        u[j] = i < hi ? __ldg(base + i) : make_uint4(0u, 0u, 0u, 0u);
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
  cluster_wait();
  if (t < T && lane < k) {
    const int p = t * k + lane;
    a.ids[p] = my_id;
    a.w[p] = my_w;
#pragma unroll
    for (int r = 0; r < kCluster; ++r) st_cluster(smem_addr(&s_ids[p]), r, static_cast<uint32_t>(my_id));
  }
  if (a.dynamic && tid < kCluster) {
    float r = 0.0f;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) r = fmaxf(r, s_red[i]);
    st_cluster(smem_addr(&s_part[c]), tid, __float_as_uint(r));
  }
  cluster_arrive();
  cluster_wait();  // all ids and partial maxima are now in this CTA's shared memory

  // ---- 2. the permutation, derived locally -----------------------------------------------
  for (int p = tid; p < P; p += kThreads) atomicOr(&s_mask[s_ids[p]], 1ull << (p / k));
  __syncthreads();
  {
    // packed per-expert triple: padded count << 32 | active flag << 16 | count (no field
    // overflows: counts sum to P <= 2048, flags to E <= 1024)
    const int mt = 1 << a.m_tile_log2;
    unsigned long long v[4], tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 4 * tid + i;
      const int cnt = e < E ? __popcll(s_mask[e]) : 0;
      const int pad = (cnt + mt - 1) >> a.m_tile_log2 << a.m_tile_log2;
      v[i] = (static_cast<unsigned long long>(pad) << 32) | (static_cast<unsigned long long>(cnt > 0) << 16) |
             static_cast<unsigned long long>(cnt);
      if (e < E) s_cnt[e] = cnt;
      tot += v[i];
    }
    unsigned long long incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    unsigned long long run = incl - tot;
    for (int i = 0; i < warp; ++i) run += s_wsum[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 4 * tid + i;
      if (e <= E) {
        s_off[e] = static_cast<int32_t>(run & 0xFFFFu);
        s_aoff[e] = static_cast<int32_t>((run >> 16) & 0xFFFFu);
        s_poff[e] = static_cast<int32_t>(run >> 32);
      }
      run += v[i];
    }
    if (tid == kThreads - 1 && E == MAX_E) {  // the grand total when E fills every slot
      s_off[E] = static_cast<int32_t>(run & 0xFFFFu);
      s_aoff[E] = static_cast<int32_t>((run >> 16) & 0xFFFFu);
      s_poff[E] = static_cast<int32_t>(run >> 32);
    }
  }
  __syncthreads();
  for (int p = tid; p < P; p += kThreads) {
    const int e = s_ids[p];
    const int tk = p / k;
    s_row[p] = s_poff[e] + __popcll(s_mask[e] & ((1ull << tk) - 1ull));
  }
  if (a.list)
    for (int e = tid; e < E; e += kThreads)
      if (s_cnt[e] > 0) s_act[s_aoff[e]] = e;
  __syncthreads();

  // ---- 3. global writes, split over the cluster ------------------------------------------
  for (int p = gi; p < P; p += kAll) {
    const int row = s_row[p];
    a.pair_to_row[p] = row;
    a.row_token[row] = p / k;
    a.row_pair[row] = p;
  }
  for (int e = gi; e < E; e += kAll) {
    a.counts[e] = s_cnt[e];
    a.offsets[e] = s_off[e];
    a.padded_offsets[e] = s_poff[e];
    if (s_cnt[e] > 0) a.active[1 + s_aoff[e]] = e;
    if (a.zero_f32) a.zero_f32[e] = 0.0f;
  }
  float s_t;
  if (a.dynamic) {
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < kCluster; ++i) mx = fmaxf(mx, s_part[i]);
    s_t = __fdiv_rn(mx, 2688.0f);
  } else {
    s_t = a.x_codes ? *a.x_scale : 0.0f;  // no x codes: the weight-only layer keeps x in bf16
  }
  if (gi == 0) {
    a.offsets[E] = s_off[E];
    a.padded_offsets[E] = s_poff[E];
    a.active[0] = s_aoff[E];
    if (a.dynamic) *a.x_scale = s_t;
  }
  if (a.list) {
    // the fused GEMM's work list: gate/up items then down items, each (active expert, weight
    // tile) with all the expert's tokens as one chunk; and its counters, zeroed
    const int na = s_aoff[E];
    const int ng = na * a.wt_gateup, nd = na * a.wt_down;
    if (gi == 0) a.list[0] = make_int4(ng, nd, 0, 0);
    for (int i = gi; i < ng + nd; i += kAll) {
      const bool g = i < ng;
      const int idx = g ? i : i - ng;
      const int wt = g ? a.wt_gateup : a.wt_down;
      const int e = s_act[idx / wt];
      a.list[1 + i] = make_int4(e, idx % wt, s_poff[e], s_cnt[e]);
    }
    for (int e = gi; e < E; e += kAll) a.done[e] = 0;
  }
  // padding rows and the tile -> expert map: one warp of the cluster per expert at a time
  for (int e = c * kWarps + warp; e < E; e += kCluster * kWarps) {
    const int p0 = s_poff[e], p1 = s_poff[e + 1];
    for (int r = p0 + s_cnt[e] + lane; r < p1; r += 32) {
      a.row_token[r] = -1;
      a.row_pair[r] = -1;
    }
    for (int tl = (p0 >> a.m_tile_log2) + lane; tl < (p1 >> a.m_tile_log2); tl += 32) a.tile_expert[tl] = e;
  }

  // quantise each 16-element block of x once; write it to its row(s)
  const int nb = H / 16;
  const int64_t rb = H / 2;
  for (int item = gi; a.x_codes && item < T * nb; item += kAll) {
    const int tk = item / nb, b = item - tk * nb;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + int64_t(tk) * H + b * 16);
    const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
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
      const int64_t row = a.expert_order ? s_row[tk * k + d] : tk;
      *reinterpret_cast<uint2*>(a.x_codes + row * rb + b * 8) = code;
      a.x_sf[sf_mma_offset(row, b, H)] = static_cast<uint8_t>(sf);
    }
  }
}

}  // namespace

bool prologue_fits(int T, int E, int k) { return T >= 1 && T <= MAX_T && E <= MAX_E && k >= 1 && k <= 32; }

nvfp4moe_status launch_prologue(const void* x, const float* logits, int T, int H, int E, int k, int m_tile,
                                int dynamic, float* x_scale, int32_t* ids, float* w, int32_t* counts, int32_t* offsets,
                                int32_t* padded_offsets, int32_t* pair_to_row, int32_t* row_token, int32_t* row_pair,
                                int32_t* tile_expert, int32_t* active, float* zero_f32, int expert_order,
                                uint8_t* x_codes, uint8_t* x_sf, int4* list, int* done, int wt_gateup, int wt_down,
                                cudaStream_t s) {
  NVFP4_REQUIRE(prologue_fits(T, E, k), NVFP4MOE_UNSUPPORTED_SHAPE, "prologue: T=%d E=%d k=%d out of range", T, E, k);
  int lg = 0;
  while ((1 << lg) < m_tile) ++lg;
  NVFP4_REQUIRE((1 << lg) == m_tile, NVFP4MOE_INVALID_ARG, "prologue: m_tile %d is not a power of two", m_tile);
  PrologueArgs a;
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
  a.list = list; a.done = done;
  a.wt_gateup = wt_gateup; a.wt_down = wt_down;
  const int per = (E + 31) / 32;
  if (per <= 1)
    prologue_kernel<1><<<kCluster, kThreads, 0, s>>>(a);
  else if (per <= 4)
    prologue_kernel<4><<<kCluster, kThreads, 0, s>>>(a);
  else if (per <= 8)
    prologue_kernel<8><<<kCluster, kThreads, 0, s>>>(a);
  else if (per <= 16)
    prologue_kernel<16><<<kCluster, kThreads, 0, s>>>(a);
  else
    prologue_kernel<32><<<kCluster, kThreads, 0, s>>>(a);
  return check_launch("prologue");
}

}  // namespace nvfp4moe
