// Weight-stationary grouped GEMM of the routed layer on tcgen05 block-scaled MMA
// (kind::mxf4nvf4, E4M3 scales per 16 elements, fp32 accumulators in TMEM).
//
// The expert weights are the MMA's M operand (128 weight rows per tile) and an expert's
// tokens are its N operand: N = the expert's token count in the tile's chunk rounded up to 16,
// at most BNMAX (64 for batches of at most 64 tokens, 192 above).  A weight tile is streamed
// once per chunk of its expert's tokens whatever the routing skew, and no MMA work or load
// is spent on 128-row padding of experts that received a handful of tokens.  One kernel
// serves decode and prefill, gate/up (EPI_GATEUP), down (EPI_DOWN) or both in one launch
// (EPI_FUSED).
//
// Persistent CTA per SM; work items ordered (expert, weight tile, token chunk) with the
// chunk fastest, so CTAs of one wave that share a weight tile run together (L2 hits).
//   warp 0      weight producer: TMA loads of 128 rows x 128 B (128-byte swizzle) and bulk
//               copies of their 512-byte scale atoms into a ring of STAGES stages; it arms
//               each stage with the bytes of both operands;
//   warp 10     token producer: TMA loads of the tokens' rows (64- and 16-row boxes) and
//               their scale atoms into the same stages (for a fused down item, once its
//               expert's gate/up tiles are counted done);
//   warp 1      TMEM owner and MMA issuer: tcgen05.cp of the scales, four K=64 MMAs per
//               stage into one of NACC fp32 accumulators;
//   warps 2..9  epilogue, two warps per 32-row TMEM lane quarter (alternate token chunks):
//               SwiGLU + requantise to NVFP4 (gate/up; gate row i and up row i are lanes i
//               and 16+i of the same warp by the W13 interleave), or the down rows scaled by
//               s_h * s_w2 into fp32 slot rows (by pair, weighted; or, above 64 tokens, by
//               padded row through staging tiles and TMA tile stores) or added into the
//               fp32 accumulator (bulk reductions).
// Scale atoms of the tokens start at a 64-row boundary inside a 128-row atom, so the MMA
// reads them at a TMEM column offset of 0 or 2.  Every wait is bounded (status bit on
// timeout; copies in flight land before the CTA exits).
#include "ffn_gemm.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace nvfp4moe {
namespace {

using namespace sm100;

constexpr int WM = 128;         // weight rows per tile
constexpr int TOK_ALIGN = 64;   // token rows per permutation block (scale atoms start at 0 or 64)
constexpr int NQ = 16;          // MMA N granularity and the small token box height
constexpr int BK = 256;
constexpr int KB = BK / 2;
constexpr int EPI_WARPS = 8;    // two per TMEM lane quarter
constexpr int TOKEN_WARP = 2 + EPI_WARPS;  // the producer of token tiles, after the epilogue warps
constexpr int kThreads = 32 * (TOKEN_WARP + 1);
constexpr uint32_t kTmemCols = 512;
constexpr int MAX_E = 1024;
constexpr uint32_t kDevTimeout = 1u << 3;
constexpr int TR_STRIDE = 17;   // h transpose tile: 32 tokens x 16 (+1) floats
constexpr int TR_FLOATS = 32 * TR_STRIDE;
constexpr int DOWN_TR_STRIDE = 33;  // down transpose tile: 16 tokens x 32 (+1) floats
static_assert(16 * DOWN_TR_STRIDE <= TR_FLOATS, "down tile fits the transpose buffer");
constexpr int SFB_PER_KB = 8;   // TMEM columns of token scales per k-block (two atoms)
constexpr int SCHED_CAP = 1264; // work items of one CTA kept as a list (over the per-expert arrays)
constexpr int SCHED_PER_THREAD = (SCHED_CAP + kThreads - 1) / kThreads;

// Tile configuration: BNMAX tokens per tile at most, STAGES shared-memory stages, NACC TMEM
// accumulators.
//   <192, 4, 2> gate/up and <192, 3, 2, tile stores> down above 64 tokens (the down epilogue
//   stores its output through per-warp staging tiles with TMA, slot rows in expert order);
//   <64, 6, 4> when no expert can hold more than 64 tokens (T <= 64): more weight bytes in
//   flight for the small decode tiles, and the MMA may run three items ahead of a slow
//   epilogue.
template <int BN_, int STAGES_, int NACC_, bool OUT_TMA_>
struct Cfg {
  static constexpr int BNMAX = BN_;
  static constexpr int STAGES = STAGES_;
  static constexpr int NACC = NACC_;                     // TMEM accumulators (items in flight)
  // down output by tile stores: two 16-token x 32-row fp32 staging tiles per epilogue warp
  static constexpr bool OUT_TMA = OUT_TMA_;
  static constexpr int OUT_TILE_BYTES = 16 * 32 * 4;
  static constexpr int OUT_BYTES = OUT_TMA ? EPI_WARPS * 2 * OUT_TILE_BYTES : 0;
  static constexpr int ACC_COLS = BNMAX;
  static constexpr int SFA_COL = NACC * ACC_COLS;        // 16 columns
  static constexpr int SFB_COL = SFA_COL + 16;           // 32 columns
  static constexpr int A_BYTES = WM * KB;                // 16 KB
  static constexpr int B_BYTES = BNMAX * KB;
  static constexpr int SFA_BYTES = WM * BK / 16;         // 2 KB
  static constexpr int SFB_BYTES = 2 * 2048;             // up to two 128-row atom rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + (2 * STAGES + 2 * NACC + 1) * 8 + 16 + (5 * MAX_E + 1) * 4 +
      EPI_WARPS * TR_FLOATS * 4 + (OUT_TMA ? 128 + OUT_BYTES : 0);
  static constexpr int MAX_CHUNKS = BNMAX / 32;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(SFB_COL + 32 <= int(kTmemCols), "TMEM budget");
};
using CfgWide = Cfg<192, 4, 2, false>;      // gate/up, batches above 64 tokens
using CfgWideDown = Cfg<192, 3, 2, true>;   // down, batches above 64 tokens (room for the tiles)
using CfgDecode = Cfg<64, 6, 4, false>;

// Modes: one GEMM per launch (gate/up or down), or both in one persistent launch (decode):
// the CTAs work through gate/up items and then down items of one list, and a down item waits
// only until every gate/up tile of its expert has written h (per-expert counters).
enum { EPI_GATEUP = 0, EPI_DOWN = 1, EPI_FUSED = 2 };

struct GroupedParams {
  int K[2];          // reduction size, per phase (0 gate/up, 1 down)
  int NW[2];         // weight rows per expert, per phase
  const uint8_t* x_sf[2];  // token scales per phase (x, h), MMA layout over the padded rows
  const uint8_t* w_sf[2];  // weight scales per phase, per expert NW*K/16 bytes
  int E;
  const int32_t* counts;
  const int32_t* padded_offsets;
  const int32_t* row_pair;
  // gate/up
  const float* x_scale;
  const float* w13_scale;
  const float* h_scale;
  float* h_amax;
  uint8_t* h_codes;
  uint8_t* h_sf;
  float* h_f32;      // nullable: dynamic h scale, h goes out in fp32 [rows][I] (and its amax)
  int I;
  // down
  const float* w2_scale;
  const float* topk_w;
  float* slots;      // [T*k][H] fp32 rows, by pair (ordered combine)
  int slots_by_row;  // tile-store configurations: slot rows in padded expert order, unweighted,
                     // written through tmO (the combine applies the routing weights)
  float* accum;      // nullable [T][H] fp32: when set, weighted rows are added here instead
  int k;             // top_k (pair -> token)
  int H;
  uint32_t* status;
  const int4* list;  // fused mode: work list written by the routing step (entry 0: {gate/up
                     // items, down items}; then the gate/up items, then the down items)
  int64_t list_cap;  // items the list can hold
  int* done;         // fused mode: per expert, epilogue warps that finished a gate/up tile
  int done_target;   // EPI_WARPS x gate/up weight tiles
};

struct Item {
  int e, mt, r0, n_rows, N, ph;
};

// Work item idx -> (expert, weight tile, token chunk); every input comes from shared memory.
// prefix[e] = items of the experts before e (experts without tokens add none).
template <int BNMAX>
__device__ __forceinline__ Item get_item(int idx, int E, const int* prefix, const int* s_ch, const int* s_off,
                                         const int* s_cnt) {
  int lo = 0, hi = E;  // the last e with prefix[e] <= idx, which has prefix[e+1] > idx
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= idx) lo = mid; else hi = mid;
  }
  Item it;
  it.e = lo;
  const int ch = s_ch[lo];
  const int rem = idx - prefix[lo];
  it.mt = rem / ch;
  const int c = rem - it.mt * ch;
  it.r0 = s_off[lo] + c * BNMAX;
  it.n_rows = min(BNMAX, s_cnt[lo] - c * BNMAX);
  it.N = (it.n_rows + NQ - 1) / NQ * NQ;
  it.ph = 0;
  return it;
}

// silu(g) * u with the fast exponential and division (h is requantised to E2M1 right after;
// a few ulp here only move values that sit on a rounding boundary of the 4-bit grid).
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// acquire load of a counter written by other CTAs (release side: fence + atomic add)
__device__ __forceinline__ int ld_acquire(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ int ld_relaxed(const int* ptr) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
__device__ __forceinline__ void red_add_v4_f32(float* p, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

template <int EPI, class C>
__global__ void __launch_bounds__(kThreads, 1)
grouped_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmX0,
               const __grid_constant__ CUtensorMap tmXs0, const __grid_constant__ CUtensorMap tmW1,
               const __grid_constant__ CUtensorMap tmX1, const __grid_constant__ CUtensorMap tmXs1,
               const __grid_constant__ CUtensorMap tmO, GroupedParams p) {
  // the phase of a single-GEMM launch; fused launches take it from each item
  constexpr int PH = EPI == EPI_DOWN ? 1 : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_shared_1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::STAGES * C::A_BYTES;
  uint8_t* sSFA = sB + C::STAGES * C::B_BYTES;
  uint8_t* sSFB = sSFA + C::STAGES * C::SFA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + C::STAGES * C::SFB_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* acc_full = bars + 2 * C::STAGES;   // [NACC]
  uint64_t* acc_empty = acc_full + C::NACC;    // [NACC]
  uint64_t* drain = acc_empty + C::NACC;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* prefix = reinterpret_cast<int*>(tmem_holder + 4);  // [MAX_E + 1]
  int* s_wsum = prefix + MAX_E + 1;                        // [8] scan partials (room for MAX_E)
  int* s_ch = s_wsum + MAX_E;                              // [MAX_E]
  int* s_off = s_ch + MAX_E;                               // [MAX_E] first padded row
  int* s_cnt = s_off + MAX_E;                              // [MAX_E] rows
  float* s_tr = reinterpret_cast<float*>(s_cnt + MAX_E);   // [EPI_WARPS][TR_FLOATS]
  // [EPI_WARPS][2] output staging tiles (tile-store configurations), 128-byte aligned
  float* s_out = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(s_tr + EPI_WARPS * TR_FLOATS) + 127) &
                                          ~uintptr_t(127));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int wtiles = p.NW[PH] / WM;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    if (EPI != EPI_DOWN) {
      prefetch_tensormap(&tmW0);
      prefetch_tensormap(&tmX0);
      prefetch_tensormap(&tmXs0);
    }
    if (EPI != EPI_GATEUP) {
      prefetch_tensormap(&tmW1);
      prefetch_tensormap(&tmX1);
      prefetch_tensormap(&tmXs1);
    }
  }
  // The expert counts and offsets come from the permutation.  Gate/up waits for the kernel
  // before it (the permutation, or the copy of x into expert order) and only then lets the
  // down launch start, so the down kernel may read the counts before its own wait.
  if (EPI != EPI_DOWN) griddep_wait();
  griddep_launch_dependents();
  int4* s_items = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(prefix) + 15) & ~uintptr_t(15));
  int total = 0, n_my = 0;
  bool sched = true;
  // Items are dealt round-robin over the fewest CTAs that keep the largest share (ceil(total /
  // grid) items): then every working CTA has the same count but for the last round, no CTA
  // carries one item more than most others, and the CTAs left over exit at once (their SMs
  // go to the next launch).
  int geff = int(gridDim.x);
  auto balance = [&](int tot) {
    if (tot > 0) {
      const int per = (tot + int(gridDim.x) - 1) / int(gridDim.x);
      geff = (tot + per - 1) / per;
    }
  };
  if (p.list != nullptr) {
    // The routing step wrote the work list (entry 0: {gate/up items, down items}, then the
    // gate/up items, then the down items).  Gate/up and fused launches read their length and
    // this CTA's entries in one round trip; a down launch first learns where its entries start.
    // The host only passes the list when a CTA's share fits SCHED_CAP.  In a fused launch the
    // entries past the gate/up items are down items; the phase goes into bit 30 of the tile.
    const int4 head = __ldcg(p.list);
    const int64_t base = EPI == EPI_DOWN ? 1 + head.x : 1;
    total = EPI == EPI_GATEUP ? head.x : EPI == EPI_DOWN ? head.y : head.x + head.y;
    balance(total);
    int4 mine[SCHED_PER_THREAD];
#pragma unroll
    for (int q = 0; q < SCHED_PER_THREAD; ++q) {
      const int j = threadIdx.x + q * kThreads;
      const int64_t idx = int64_t(blockIdx.x) + int64_t(j) * geff;
      mine[q] = (j < SCHED_CAP && idx < p.list_cap && idx < total) ? __ldcg(p.list + base + idx)
                                                                    : make_int4(0, 0, 0, 0);
    }
    n_my = int(blockIdx.x) < geff && total > int(blockIdx.x) ? (total - int(blockIdx.x) + geff - 1) / geff : 0;
#pragma unroll
    for (int q = 0; q < SCHED_PER_THREAD; ++q) {
      const int j = threadIdx.x + q * kThreads;
      const int idx = int(blockIdx.x) + j * geff;
      if (j < n_my) {
        int4 v = mine[q];
        if (EPI == EPI_FUSED) v.y |= int(idx >= head.x) << 30;
        s_items[j] = v;
      }
    }
  } else {
    // counts and first padded rows of all experts, every load in flight at once; thread t < 256
    // owns experts 4t .. 4t+3, whose item counts (chunks x weight tiles) one block scan sums
    int tot = 0, nit[4];
    if (threadIdx.x < MAX_E / 4) {
      int c[4], o[4];
  #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = 4 * int(threadIdx.x) + i;
        c[i] = e < E ? __ldcg(p.counts + e) : 0;
        o[i] = e < E ? __ldcg(p.padded_offsets + e) : 0;
      }
  #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = 4 * int(threadIdx.x) + i;
        const int ch = (c[i] + C::BNMAX - 1) / C::BNMAX;
        nit[i] = ch * wtiles;
        tot += nit[i];
        if (e < E) {
          s_cnt[e] = c[i];
          s_off[e] = o[i];
          s_ch[e] = ch;
        }
      }
    }
    int incl = tot;
  #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31 && warp < MAX_E / 128) s_wsum[warp] = incl;
    __syncthreads();
    if (threadIdx.x < MAX_E / 4) {
      int run = incl - tot;
      for (int w = 0; w < warp; ++w) run += s_wsum[w];
  #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = 4 * int(threadIdx.x) + i;
        if (e <= E) prefix[e] = run;
        run += nit[i];
      }
      if (threadIdx.x == MAX_E / 4 - 1 && E == MAX_E) prefix[E] = run;
    }
    __syncthreads();
    // This CTA's items are blockIdx.x + j * geff.  Each thread resolves a few of them now, in
    // parallel, and the list replaces the per-expert arrays, so that every role then reads one
    // 16-byte entry per item instead of searching the expert prefix sums.
    total = prefix[E];
    balance(total);
    n_my = int(blockIdx.x) < geff && total > int(blockIdx.x) ? (total - int(blockIdx.x) + geff - 1) / geff : 0;
    sched = n_my <= SCHED_CAP;
    if (sched) {
      int4 mine[SCHED_PER_THREAD];
  #pragma unroll
      for (int q = 0; q < SCHED_PER_THREAD; ++q) {
        const int j = threadIdx.x + q * kThreads;
        if (j < n_my) {
          const Item w = get_item<C::BNMAX>(int(blockIdx.x) + j * geff, E, prefix, s_ch, s_off, s_cnt);
          mine[q] = make_int4(w.e, w.mt, w.r0, w.n_rows);
        }
      }
      __syncthreads();
  #pragma unroll
      for (int q = 0; q < SCHED_PER_THREAD; ++q) {
        const int j = threadIdx.x + q * kThreads;
        if (j < n_my) s_items[j] = mine[q];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  auto item_at = [&](int j) -> Item {
    if (sched) {
      const int4 v = s_items[j];
      Item w;
      w.e = v.x; w.mt = v.y & 0xFFFF; w.r0 = v.z; w.n_rows = v.w;
      w.N = (v.w + NQ - 1) / NQ * NQ;
      w.ph = EPI == EPI_FUSED ? (v.y >> 30) & 1 : PH;
      return w;
    }
    Item w = get_item<C::BNMAX>(int(blockIdx.x) + j * geff, E, prefix, s_ch, s_off, s_cnt);
    w.ph = PH;
    return w;
  };
  auto k_tiles_of = [&](int ph) { return (p.K[ph] + BK - 1) / BK; };
  auto abort_now = [&]() {
    *abort_flag = 1;
    atomicOr(p.status, kDevTimeout);
  };

  if (warp == 0) {
    // ----------------------------------------------------- producer: weights ----
    // Weight tiles and their scales need nothing from earlier kernels (the item list was
    // written before the preceding launch let this one start), so this warp never waits on
    // them; it arms each stage with the bytes of both halves.
    if (elect_one()) {
      uint32_t it = 0;
      for (int j = 0; j < n_my && !*abort_flag; ++j) {
        const Item w = item_at(j);
        const int ph = w.ph;
        const int K = p.K[ph], NW = p.NW[ph], kt_n = k_tiles_of(ph);
        const int64_t katoms = K / 64;
        const CUtensorMap* mW = ph ? &tmW1 : &tmW0;
        const uint8_t* wsf = p.w_sf[ph] + int64_t(w.e) * NW * (K / 16);
        const int natoms = (w.r0 + w.N - 1) / 128 - w.r0 / 128 + 1;
        for (int kt = 0; kt < kt_n; ++kt, ++it) {
          const int s = it % C::STAGES;
          const uint32_t sfb = min(4, (K - kt * BK) / 64) * 512;
          if (!mbar_wait(&empty[s], ((it / C::STAGES) & 1) ^ 1)) {
            abort_now();
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::A_BYTES + w.N * KB + sfb * (1 + natoms));
          tma_load_2d(sA + s * C::A_BYTES, mW, kt * KB, w.e * NW + w.mt * WM, &full[s]);
          bulk_load(sSFA + s * C::SFA_BYTES, wsf + (int64_t(w.mt) * katoms + kt * 4) * 512, sfb, &full[s]);
        }
      }
      if (*abort_flag) {  // let the copies in flight land before the CTA exits
        for (uint32_t back = 0; back < C::STAGES && back < it; ++back) {
          const uint32_t jj = it - 1 - back;
          mbar_wait(&full[jj % C::STAGES], (jj / C::STAGES) & 1, 1u << 16);
        }
      }
    }
  } else if (warp == TOKEN_WARP) {
    // ------------------------------------------------------ producer: tokens ----
    // Token tiles and their scales are the previous kernel's output (down: h), or, fused, the
    // h rows that gate/up epilogues of this launch write: a down item's first stage waits until
    // every gate/up epilogue warp of its expert has counted itself done.  The counters of this
    // CTA's next down items are read in one round trip (relaxed loads, then one acquire fence)
    // and kept as a bit mask.  The copies complete bytes on the stage barrier that the weight
    // producer arms (a stage may receive them first).
    if (elect_one()) {
      if (EPI == EPI_DOWN) griddep_wait();
      uint64_t ready = 0;
      int ready_base = -1;
      auto ensure_ready = [&](int j, int e) -> bool {
        if (ready_base >= 0 && j >= ready_base && j < ready_base + 64 && ((ready >> (j - ready_base)) & 1)) return true;
        ready_base = j;
        ready = 0;
        int v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = j + i < n_my ? ld_relaxed(p.done + item_at(j + i).e) : 0;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (j + i < n_my && v[i] >= p.done_target) ready |= 1ull << i;
        fence_acq_rel_gpu();
        if (!(ready & 1ull)) {
          const uint64_t t0 = global_ns();
          while (ld_acquire(p.done + e) < p.done_target)
            if (global_ns() - t0 > 200000000ull) return false;  // 0.2 s: a gate/up tile never finished
          ready |= 1ull;
        }
        fence_proxy_async_global();
        return true;
      };
      uint32_t it = 0;
      for (int j = 0; j < n_my && !*abort_flag; ++j) {
        const Item w = item_at(j);
        const int ph = w.ph;
        const int K = p.K[ph], kt_n = k_tiles_of(ph);
        const int64_t katoms = K / 64;
        const CUtensorMap* mX = ph ? &tmX1 : &tmX0;
        const CUtensorMap* mXs = ph ? &tmXs1 : &tmXs0;
        const uint8_t* xsf = p.x_sf[ph];
        const int a0 = w.r0 / 128;
        const int natoms = (w.r0 + w.N - 1) / 128 - a0 + 1;
        if (EPI == EPI_FUSED && ph == 1 && !ensure_ready(j, w.e)) {
          abort_now();
          break;
        }
        for (int kt = 0; kt < kt_n; ++kt, ++it) {
          const int s = it % C::STAGES;
          const uint32_t sfb = min(4, (K - kt * BK) / 64) * 512;
          if (!mbar_wait(&empty[s], ((it / C::STAGES) & 1) ^ 1)) {
            abort_now();
            break;
          }
          int b = 0;
          for (; b + TOK_ALIGN <= w.N; b += TOK_ALIGN)
            tma_load_2d(sB + s * C::B_BYTES + b * KB, mX, kt * KB, w.r0 + b, &full[s]);
          for (; b < w.N; b += NQ) tma_load_2d(sB + s * C::B_BYTES + b * KB, mXs, kt * KB, w.r0 + b, &full[s]);
          for (int ar = 0; ar < natoms; ++ar)
            bulk_load(sSFB + s * C::SFB_BYTES + ar * 2048, xsf + (int64_t(a0 + ar) * katoms + kt * 4) * 512, sfb,
                      &full[s]);
        }
      }
      if (*abort_flag) {
        for (uint32_t back = 0; back < C::STAGES && back < it; ++back) {
          const uint32_t jj = it - 1 - back;
          mbar_wait(&full[jj % C::STAGES], (jj / C::STAGES) & 1, 1u << 16);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA ----
    if (elect_one()) {
      uint32_t it = 0, li = 0;
      for (int j = 0; j < n_my && !*abort_flag; ++j, ++li) {
        const Item w = item_at(j);
        const uint32_t ab = li % C::NACC;
        if (!mbar_wait(&acc_empty[ab], ((li / C::NACC) & 1) ^ 1)) {
          abort_now();
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_mxf4nvf4(WM, w.N);
        const int natoms = (w.r0 + w.N - 1) / 128 - w.r0 / 128 + 1;
        const uint32_t g0 = (w.r0 % 128) / 32;  // 0 or 2
        const uint32_t d_acc = tmem + ab * C::ACC_COLS;
        bool ok = true;
        const int kt_n = k_tiles_of(w.ph), K = p.K[w.ph];
        for (int kt = 0; kt < kt_n; ++kt, ++it) {
          const int s = it % C::STAGES;
          if (!mbar_wait(&full[s], (it / C::STAGES) & 1)) {
            abort_now();
            ok = false;
            break;
          }
          tc_fence_after();
          const int nkb = min(4, (K - kt * BK) / 64);
          // descriptor start addresses advance in 16-byte units: 512-byte atoms (32), 32 bytes of K (2)
          const uint64_t sfa_d = desc_sf_atom(sSFA + s * C::SFA_BYTES);
          const uint64_t sfb_d = desc_sf_atom(sSFB + s * C::SFB_BYTES);
          const uint64_t a_d = desc_kmajor_sw128(sA + s * C::A_BYTES);
          const uint64_t b_d = desc_kmajor_sw128(sB + s * C::B_BYTES);
          if (nkb == 4) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tc_cp_sf(tmem + C::SFA_COL + 4 * j, sfa_d + 32 * j);
              tc_cp_sf(tmem + C::SFB_COL + SFB_PER_KB * j, sfb_d + 32 * j);
              if (natoms > 1) tc_cp_sf(tmem + C::SFB_COL + SFB_PER_KB * j + 4, sfb_d + 128 + 32 * j);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc_mma_mxf4nvf4(d_acc, a_d + 2 * j, b_d + 2 * j, idesc, tmem + C::SFA_COL + 4 * j,
                              tmem + C::SFB_COL + SFB_PER_KB * j + g0, (kt | j) != 0 ? 1u : 0u);
          } else {
            for (int j = 0; j < nkb; ++j) {
              tc_cp_sf(tmem + C::SFA_COL + 4 * j, sfa_d + 32 * j);
              for (int ar = 0; ar < natoms; ++ar)
                tc_cp_sf(tmem + C::SFB_COL + SFB_PER_KB * j + 4 * ar, sfb_d + 128 * ar + 32 * j);
            }
            for (int j = 0; j < nkb; ++j)
              tc_mma_mxf4nvf4(d_acc, a_d + 2 * j, b_d + 2 * j, idesc, tmem + C::SFA_COL + 4 * j,
                              tmem + C::SFB_COL + SFB_PER_KB * j + g0, (kt | j) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&acc_full[ab]);
      }
      tc_commit(drain);
      mbar_wait(drain, 0, 1u << 20);
    }
  } else {
    // ------------------------------------------------------------ epilogue ----
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;       // the two warps of a quarter split the token chunks
    const uint32_t trow = tmem + (uint32_t(q * 32) << 16);
    float* tr = s_tr + (warp - 2) * TR_FLOATS;
    uint32_t li = 0;
    // Fused: this warp's h stores of a gate/up tile are counted for the expert's down items one
    // item later (or at the end), so the fence that orders them before the count finds them
    // drained instead of stalling the epilogue.
    int pending = -1;
    // down output through staging tiles and tile stores (slot rows in expert order, unweighted)
    const bool tile_out = C::OUT_TMA && p.slots_by_row && p.accum == nullptr;
    // accumulating with the staging tiles: each token's 32 weighted rows are added into its
    // output row by one bulk reduction (L2 performs the fp32 adds)
    const bool tile_red = C::OUT_TMA && p.accum != nullptr;
    float* out_tiles = s_out + (warp - 2) * 2 * (C::OUT_TILE_BYTES / 4);
    uint32_t out_seq = 0;  // tile stores this warp has issued
    auto release_pending = [&]() {
      if (EPI == EPI_FUSED && pending >= 0) {
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.done + pending, 1);
        pending = -1;
      }
    };
    for (int j = 0; j < n_my && !*abort_flag; ++j, ++li) {
      const Item w = item_at(j);
      const uint32_t ab = li % C::NACC;
      const int wrow = w.mt * WM + q * 32 + lane;  // this lane's weight row inside the expert
      // per-item data, fetched before the accumulator is ready so its latency is hidden
      float sg = 0.f, su = 0.f, sh = 0.f, sc = 0.f;
      int32_t pr[C::MAX_CHUNKS / 2];
      float wt[C::MAX_CHUNKS / 2];
      const bool gateup = EPI == EPI_FUSED ? w.ph == 0 : EPI == EPI_GATEUP;
      if (gateup) {
        const float sx = p.x_scale[0];
        sg = sx * p.w13_scale[2 * w.e];
        su = sx * p.w13_scale[2 * w.e + 1];
        sh = p.h_scale[w.e];
      } else {
        sc = p.h_scale[w.e] * p.w2_scale[w.e];
        if (!tile_out) {
#pragma unroll
          for (int c2 = 0; c2 < C::MAX_CHUNKS / 2; ++c2) {
            const int tok = (2 * c2 + half) * 32 + lane;
            pr[c2] = tok < w.n_rows ? p.row_pair[w.r0 + tok] : -1;
          }
#pragma unroll
          for (int c2 = 0; c2 < C::MAX_CHUNKS / 2; ++c2) wt[c2] = pr[c2] >= 0 ? p.topk_w[pr[c2]] * sc : 0.0f;
        }
      }
      release_pending();
      if (!mbar_wait(&acc_full[ab], (li / C::NACC) & 1)) {
        abort_now();
        break;
      }
      tc_fence_after();
      if (gateup) {
        // lanes 0..15 hold gate rows i, lanes 16..31 the up rows i of one 16-wide block of h
        const int64_t iblk = wrow >> 5;
        float amax_all = 0.0f;
#pragma unroll 1
        for (int cc = half; cc * 32 < w.N; cc += 2) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(trow + ab * C::ACC_COLS + cc * 32, r);
          tmem_ld_wait();
          // lane l < 16 finishes tokens 0..15 of gate/up row pair l, lane l + 16 tokens 16..31
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float mine_lo = __uint_as_float(r[j]), mine_hi = __uint_as_float(r[16 + j]);
            const float other = __shfl_xor_sync(0xffffffffu, lane < 16 ? mine_hi : mine_lo, 16);
            const float g = lane < 16 ? mine_lo : other;
            const float u = lane < 16 ? other : mine_hi;
            tr[(j + 16 * (lane >> 4)) * TR_STRIDE + (lane & 15)] = silu_mul(g * sg, u * su);
          }
          __syncwarp();
          // lane t quantises token t's 16 values (one block) in-thread
          float hb[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) hb[i] = tr[lane * TR_STRIDE + i];
          __syncwarp();
          const int tok = cc * 32 + lane;
          if (tok < w.n_rows) {
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(hb[i]));
            const int64_t row = int64_t(w.r0) + tok;
            if (p.h_f32) {
              // dynamic h scale: the block goes out in fp32; it is requantised once the
              // expert's amax over the whole call is known
              float4* dst = reinterpret_cast<float4*>(p.h_f32 + row * p.I + iblk * 16);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_float4(hb[4 * i], hb[4 * i + 1], hb[4 * i + 2], hb[4 * i + 3]);
            } else {
              float inv;
              const uint32_t sf = block_scale(amax, sh, &inv);
              *reinterpret_cast<uint2*>(p.h_codes + row * (p.I / 2) + iblk * 8) = encode_block16(hb, inv);
              p.h_sf[sf_mma_offset(row, iblk, p.I)] = static_cast<uint8_t>(sf);
            }
            amax_all = fmaxf(amax_all, amax);
          }
        }
        if (p.h_amax) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) amax_all = fmaxf(amax_all, __shfl_xor_sync(0xffffffffu, amax_all, o));
          if (lane == 0 && amax_all > 0.0f) atomicMax(reinterpret_cast<int*>(p.h_amax + w.e), __float_as_int(amax_all));
        }
        if (EPI == EPI_FUSED) pending = w.e;  // counted once its stores have drained
      } else {
        if (tile_out) {
          // Each 16-token half of a chunk: this quarter's 32 rows x 16 tokens, scaled by
          // s_h * s_w2, are parked row-major in one of the warp's two staging tiles and stored
          // by one lane with a tile store into the tokens' slot rows (expert order), which the
          // combine weights and sums.  A tile is rewritten only once the store issued from it
          // two steps earlier has read it.
#pragma unroll 1
          for (int c2 = 0; c2 < C::MAX_CHUNKS / 2; ++c2) {
            const int cc = 2 * c2 + half;
            if (cc * 32 >= w.N) break;
            uint32_t r[32];
            tmem_ld_32x32b_x32(trow + ab * C::ACC_COLS + cc * 32, r);
            tmem_ld_wait();
            const int nj = min(32, w.n_rows - cc * 32);
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
              if (sub * 16 >= nj) break;
              float* tile = out_tiles + (out_seq & 1u) * (C::OUT_TILE_BYTES / 4);
              if (lane == 0 && out_seq >= 2) bulk_wait_group_read<1>();
              __syncwarp();
#pragma unroll
              for (int t = 0; t < 16; ++t) tile[t * 32 + lane] = __uint_as_float(r[sub * 16 + t]) * sc;
              fence_proxy_async_shared();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tmO, w.mt * WM + q * 32, w.r0 + cc * 32 + sub * 16, tile);
                bulk_commit_group();
              }
              ++out_seq;
            }
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[ab]);
          continue;
        }
        if (tile_red) {
          // As above, but each row is scaled by its token's routing weight and lanes 0..15
          // each add one token's 32 values (128 bytes) into the token's accumulator row.
#pragma unroll 1
          for (int c2 = 0; c2 < C::MAX_CHUNKS / 2; ++c2) {
            const int cc = 2 * c2 + half;
            if (cc * 32 >= w.N) break;
            uint32_t r[32];
            tmem_ld_32x32b_x32(trow + ab * C::ACC_COLS + cc * 32, r);
            tmem_ld_wait();
            const int nj = min(32, w.n_rows - cc * 32);
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
              if (sub * 16 >= nj) break;
              float* tile = out_tiles + (out_seq & 1u) * (C::OUT_TILE_BYTES / 4);
              if (out_seq >= 2) bulk_wait_group_read<1>();
              __syncwarp();
#pragma unroll
              for (int t = 0; t < 16; ++t)
                tile[t * 32 + lane] = __uint_as_float(r[sub * 16 + t]) * __shfl_sync(0xffffffffu, wt[c2], sub * 16 + t);
              fence_proxy_async_shared();
              __syncwarp();
              const int32_t pair = __shfl_sync(0xffffffffu, pr[c2], sub * 16 + (lane & 15));
              if (lane < 16 && pair >= 0)
                bulk_reduce_add_f32(p.accum + int64_t(pair / p.k) * p.H + int64_t(w.mt) * WM + q * 32, tile + lane * 32,
                                    128u);
              bulk_commit_group();
              ++out_seq;
            }
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[ab]);
          continue;
        }
        // A chunk's 32 token columns go through the warp's transpose tile in two halves of 16
        // tokens: lanes (= weight rows) park their accumulators, then each store instruction of
        // the warp covers 4 tokens x the quarter's 32 rows, 128 contiguous bytes per token
        // (lane l: token l >> 3 of the step, rows 4 * (l & 7) .. +4), scaled by the token's
        // routing weight.  The rows go to the token's fp32 slot row, or, accumulating, are
        // added into its output row.
        const int tq = lane >> 3, cq = lane & 7;
#pragma unroll
        for (int c2 = 0; c2 < C::MAX_CHUNKS / 2; ++c2) {
          const int cc = 2 * c2 + half;
          if (cc * 32 >= w.N) break;
          uint32_t r[32];
          tmem_ld_32x32b_x32(trow + ab * C::ACC_COLS + cc * 32, r);
          tmem_ld_wait();
          const int nj = min(32, w.n_rows - cc * 32);
          if (nj <= 8) {
            // a few tokens (decode): each token's 32 rows are one 128-byte access of the warp
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (j >= nj) break;
              const int32_t pair = __shfl_sync(0xffffffffu, pr[c2], j);
              const float wj = __shfl_sync(0xffffffffu, wt[c2], j);
              if (pair >= 0) {
                const float v = __uint_as_float(r[j]) * wj;
                if (p.accum) red_add_f32(p.accum + int64_t(pair / p.k) * p.H + wrow, v);
                else p.slots[int64_t(pair) * p.H + wrow] = v;
              }
            }
            continue;
          }
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            if (sub * 16 >= nj) break;
#pragma unroll
            for (int t = 0; t < 16; ++t) tr[t * DOWN_TR_STRIDE + lane] = __uint_as_float(r[sub * 16 + t]);
            __syncwarp();
#pragma unroll
            for (int st = 0; st < 4; ++st) {
              const int tok = 4 * st + tq;
              const int32_t pair = __shfl_sync(0xffffffffu, pr[c2], sub * 16 + tok);
              const float wj = __shfl_sync(0xffffffffu, wt[c2], sub * 16 + tok);
              const float* src = tr + tok * DOWN_TR_STRIDE + 4 * cq;
              const float4 v = make_float4(src[0] * wj, src[1] * wj, src[2] * wj, src[3] * wj);
              if (pair >= 0) {
                const int64_t col = int64_t(w.mt) * WM + q * 32 + 4 * cq;
                if (p.accum) red_add_v4_f32(p.accum + int64_t(pair / p.k) * p.H + col, v);
                else *reinterpret_cast<float4*>(p.slots + int64_t(pair) * p.H + col) = v;
              }
            }
            __syncwarp();
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
    release_pending();
    if ((tile_out && lane == 0) || tile_red) bulk_wait_group<0>();  // the bulk writes are complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

struct Maps {
  CUtensorMap w, x, xs;
};

template <int EPI, class C>
nvfp4moe_status launch_cfg(const Maps& m0, const Maps& m1, const CUtensorMap& out, const GroupedParams& p,
                           int64_t max_items, cudaStream_t s) {
  auto kern = grouped_kernel<EPI, C>;
  {
    const cudaError_t e = set_smem_limit_once<grouped_kernel<EPI, C>>(C::SMEM_BYTES);
    if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "grouped GEMM smem attribute: %s", cudaGetErrorString(e));
  }
  int64_t grid = num_sms();
  if (max_items < grid) grid = max_items > 0 ? max_items : 1;
  const cudaError_t e = launch_dependent(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), C::SMEM_BYTES, s,
                                         m0.w, m0.x, m0.xs, m1.w, m1.x, m1.xs, out, p);
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "grouped tcgen05 GEMM: %s", cudaGetErrorString(e));
  return check_launch("grouped tcgen05 GEMM");
}

// upper bound of one GEMM's work items: every expert its token chunks, weight tiles per chunk
int64_t max_items(int64_t P, int64_t E, int64_t bn, int64_t weight_tiles) {
  return ((P < E ? P : E) + P / bn + 1) * weight_tiles;
}

}  // namespace

int grouped_token_align() { return TOK_ALIGN; }

int64_t grouped_fused_list_entries(int64_t active_max, int64_t wt_gateup, int64_t wt_down) {
  return 1 + active_max * (wt_gateup + wt_down);
}

nvfp4moe_status launch_grouped_ffn(const GemmFfnArgs& a, cudaStream_t s) {
  uint32_t* status = device_status_ptr();
  if (!status) return fail(NVFP4MOE_CUDA_ERROR, "device status word unavailable");
  if (a.E > MAX_E) return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "grouped GEMM: E > %d", MAX_E);
  const int64_t P = int64_t(a.T) * a.k;
  // no expert receives more than T tokens (a token names an expert at most once)
  const bool decode = a.T <= CfgDecode::BNMAX;
  const int wt_g = 2 * a.I / WM, wt_d = a.H / WM;
  Maps g, d;
  // gate/up: weights W13 [E*2I][H], tokens x [rows_cap][H]; down: W2 [E*H][I], tokens h [rows_cap][I]
  nvfp4moe_status st = make_code_map(&g.w, a.w13_codes, int64_t(a.E) * 2 * a.I, a.H, WM);
  if (st == NVFP4MOE_OK) st = make_code_map(&g.x, a.x_codes, a.rows_cap, a.H, TOK_ALIGN);
  if (st == NVFP4MOE_OK) st = make_code_map(&g.xs, a.x_codes, a.rows_cap, a.H, NQ);
  if (st == NVFP4MOE_OK) st = make_code_map(&d.w, a.w2_codes, int64_t(a.E) * a.H, a.I, WM);
  if (st == NVFP4MOE_OK) st = make_code_map(&d.x, a.h_codes, a.rows_cap, a.I, TOK_ALIGN);
  if (st == NVFP4MOE_OK) st = make_code_map(&d.xs, a.h_codes, a.rows_cap, a.I, NQ);
  if (st != NVFP4MOE_OK) return st;
  GroupedParams p{};
  p.E = a.E;
  p.counts = a.counts;
  p.padded_offsets = a.padded_offsets;
  p.row_pair = a.row_pair;
  p.status = status;
  p.K[0] = a.H;
  p.NW[0] = 2 * a.I;
  p.x_sf[0] = a.x_sf;
  p.w_sf[0] = a.w13_sf;
  p.K[1] = a.I;
  p.NW[1] = a.H;
  p.x_sf[1] = a.h_sf;
  p.w_sf[1] = a.w2_sf;
  p.x_scale = a.x_scale;
  p.w13_scale = a.w13_scale;
  p.h_scale = a.h_scale;
  p.h_amax = a.h_amax;
  p.h_codes = a.h_codes;
  p.h_sf = a.h_sf;
  p.h_f32 = a.h_f32;
  p.I = a.I;
  p.w2_scale = a.w2_scale;
  p.topk_w = a.topk_w;
  p.slots = static_cast<float*>(a.slots_f32);
  p.accum = a.accum;
  // wide tiling, ordered combine: the down epilogue stores tiles into slot rows in expert order
  CUtensorMap out_map = d.w;  // unused unless tile stores are on
  p.slots_by_row = (!decode && a.slots_by_row && a.accum == nullptr) ? 1 : 0;
  if (p.slots_by_row) {
    st = make_f32_rows_map(&out_map, a.slots_f32, a.rows_cap, a.H, 32, 16);
    if (st != NVFP4MOE_OK) return st;
  }
  p.k = a.k;
  p.H = a.H;
  auto mark4 = [&]() -> nvfp4moe_status {
    if (!a.stage_events) return NVFP4MOE_OK;
    const cudaError_t e = record_mark(a.stage_events[4], s);
    return e == cudaSuccess ? NVFP4MOE_OK : fail(NVFP4MOE_CUDA_ERROR, "stage mark 4: %s", cudaGetErrorString(e));
  };

  // Decode batches with a work list from the routing step: both GEMMs in one launch, when
  // every CTA's share of the list fits the shared-memory list.
  const int64_t items_g = max_items(P, a.E, CfgDecode::BNMAX, wt_g), items_d = max_items(P, a.E, CfgDecode::BNMAX, wt_d);
  const int64_t fused_items = items_g + items_d;
  const int64_t fused_grid = fused_items < num_sms() ? fused_items : num_sms();
  // One launch pays off when the down GEMM has no more weight tiles than gate/up (H <= 2I):
  // then a second launch's ramp-up is not amortised.  Otherwise the down launch starts on the
  // SMs that gate/up frees and streams its first weight tiles meanwhile.
  const bool fits = [&](int64_t cap, int64_t grid) { return (cap + grid - 1) / grid <= SCHED_CAP; }(
      a.list_cap, fused_grid);
  auto requant = [&]() -> nvfp4moe_status {
    return a.h_f32 ? launch_requant_h(a.h_f32, a.rows_cap, a.I, a.E, a.padded_offsets, a.row_pair, a.tile_expert,
                                      a.m_tile_log2, a.h_amax, a.h_amax_user, const_cast<float*>(a.h_scale), a.h_codes,
                                      a.h_sf, s)
                   : NVFP4MOE_OK;
  };
  if (decode && a.list != nullptr && a.done != nullptr && wt_d <= wt_g && fits && a.h_f32 == nullptr) {
    p.list = a.list;
    p.list_cap = a.list_cap;
    p.done = a.done;
    p.done_target = EPI_WARPS * wt_g;
    st = launch_cfg<EPI_FUSED, CfgDecode>(g, d, out_map, p, fused_items, s);
    if (st != NVFP4MOE_OK) return st;
    return mark4();  // one launch: the gate/up stage holds both GEMMs
  }
  if (decode) {
    const int64_t cap_g = a.list_cap / (wt_g + wt_d) * wt_g, cap_d = a.list_cap - cap_g;
    const int64_t grid_g = items_g < num_sms() ? items_g : num_sms(), grid_d = items_d < num_sms() ? items_d : num_sms();
    const bool use = a.list != nullptr && (cap_g + grid_g - 1) / grid_g <= SCHED_CAP &&
                     (cap_d + grid_d - 1) / grid_d <= SCHED_CAP;
    p.list = use ? a.list : nullptr;
    p.list_cap = cap_g;
    st = launch_cfg<EPI_GATEUP, CfgDecode>(g, g, out_map, p, items_g, s);
    if (st == NVFP4MOE_OK) st = mark4();
    if (st == NVFP4MOE_OK) st = requant();
    p.list_cap = cap_d;
    if (st == NVFP4MOE_OK) st = launch_cfg<EPI_DOWN, CfgDecode>(d, d, out_map, p, items_d, s);
    return st;
  }
  st = launch_cfg<EPI_GATEUP, CfgWide>(g, g, out_map, p, max_items(P, a.E, CfgWide::BNMAX, wt_g), s);
  if (st == NVFP4MOE_OK) st = mark4();
  if (st == NVFP4MOE_OK) st = requant();
  if (st == NVFP4MOE_OK)
    st = launch_cfg<EPI_DOWN, CfgWideDown>(d, d, out_map, p, max_items(P, a.E, CfgWideDown::BNMAX, wt_d), s);
  return st;
}

}  // namespace nvfp4moe
