// The whole routed layer in ONE persistent launch for batches of at most 16 tokens (decode,
// and the dense layer at T = 1): routing, permutation, x quantisation, gate/up + SwiGLU +
// requantisation, down and the ordered combine.
//
// At decode sizes the layer is a stream of expert weights (about 1.69 MB per touched expert
// at H2048/I512) with a few kilobytes of activations, so its time is the weight bytes over
// HBM bandwidth plus whatever latency precedes and follows the stream.  This kernel keeps
// that latency to one launch:
//
//  * Every CTA routes the whole batch itself (warp t takes token t, its logits requested at
//    kernel entry), derives the permutation and the work list locally, and starts streaming
//    its first weight tiles at once.  No kernel before it computes anything, so nothing has
//    to be waited for before the stream.
//  * Every CTA quantises the whole of x (dynamic tensor scale amax / 2688 over the batch)
//    into shared memory, in the 128-byte-swizzled K-major layout the MMA reads, with the
//    block scales staged once into TMEM.  x itself arrives by one bulk copy at entry, into
//    the weight ring, which no tile uses before the routing is done (when x does not fit
//    there, the epilogue warps load and quantise it once the stream has started).  The gate/up MMA takes ALL T tokens (padded to the
//    MMA's N = 16) as its B operand for every expert: one weight tile times the resident
//    token tile.  Each output column depends only on its own token, so the columns of the
//    tokens an expert did not receive are simply not used; the extra MMA work is free at
//    this size, and no token tile is loaded per item.
//  * Two schedules of the weight tiles, chosen per call from the routing (every CTA takes the
//    same decision):
//    - expert-local: units of (active expert, kcl columns of h; kcl 256, 512 or 1024),
//      round-robin over the CTAs.  A CTA runs a unit's kcl / 64 gate/up tiles (W13 rows of
//      those columns), requantises the h chunk into shared memory (K-major, 128-byte swizzle:
//      the down MMA's B operand, 16 token rows) and runs the unit's down tiles (all H rows of
//      W2, K = the chunk) from it.  No h crosses CTAs, so nothing waits on another CTA until
//      the combine; the next unit's gate/up tiles are issued before this unit's down tiles,
//      so the MMA has work while the epilogue requantises, and two h buffers alternate.
//      Taken when I % 256 == 0 and the units fill the grid's rounds to at least 80 %
//      (lf_local_width).
//    - tile-level: gate/up tiles (expert, 128 rows of W13 = 64 columns of h) and down tiles
//      (expert, K chunk of at most 2048, 128 rows of W2) spread over all CTAs.  A down tile's
//      h rows are the requantised outputs of the gate/up tiles of its expert and K chunk,
//      written to global memory (L2) by whichever CTAs ran them; per-(expert, chunk)
//      counters order the two (release: fence + atomic add; acquire: a load, then the proxy
//      fence before TMA reads h).  The weight tiles themselves never wait: the producer
//      streams W2 while h is finishing.
//  * Combine: the down epilogue writes each routed pair's weighted fp32 rows (one row per K
//    chunk) to its slots.  Tile-level: one ticket per (token, 32 output columns) and down
//    tile; the warp that takes a token's last ticket sums its k x chunks rows in slot order
//    and rounds once to bf16 (the sums are spread over the run).  Expert-local: after a
//    grid-wide barrier (one release per CTA; the launch is cooperative, so all CTAs are
//    resident) every CTA sums a slice of the [T][H] outputs the same way.
//
// A small launch before this one zeroes the counters, tickets and barrier; this kernel is its
// programmatic dependent and waits for it only before touching them (well after its start).
//
// Warp roles after the routing phase (all 16 warps route, one token each, and quantise x
// when it was staged):
//   warp 0      weight producer: TMA loads of 128 x 128-byte tiles (128-byte swizzle) and the
//               bulk copies of their scale atoms into a ring of stages;
//   warp 1      TMEM owner and MMA issuer: tcgen05.cp of the scales, four K=64 block-scaled
//               MMAs (kind::mxf4nvf4, M = 128, N = 16) per stage into one of 8 accumulators;
//   warps 2..9  epilogue: four warps (one per 32-lane TMEM quarter) per item, the two sets of
//               four taking alternate items;
//   warp 10     h producer (tile-level schedule): for down tiles, acquires the expert's chunk
//               counter and loads the h rows and their scale atoms into the stage the weight
//               producer armed;
//   warps 10-15 the inspection copies of the routing and of x (warp 10 also the h producer);
//   warps 2-15  x quantisation from global memory when x was not staged.
// Every wait is bounded (status bit on timeout; copies in flight land before the CTA exits).
#include <cmath>

#include "ffn_gemm.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"
#include "topk.cuh"

namespace nvfp4moe {
namespace {

using namespace sm100;

constexpr int LF_WARPS = 16;
constexpr int LF_THREADS = 32 * LF_WARPS;
constexpr int LF_MAXT = 16;             // tokens = the MMA's N (one 16-row token tile)
constexpr int LF_MAXE = 1024;
constexpr int LF_MAXP = LF_MAXT * 32;   // pairs: top_k <= 32
constexpr int WM = 128;                 // weight rows per tile (the MMA's M)
constexpr int BK = 256;                 // K per stage
constexpr int KB = BK / 2;              // bytes per row per stage
constexpr int TOK_ALIGN = 64;           // padded rows per active expert (h and the x copies)
constexpr int EPI_FIRST = 2, EPI_WARPS = 8, HPROD_WARP = 10;  // warps 11..15: set-up only
constexpr int NACC = 8;                 // TMEM accumulators (items in flight past the MMA)
constexpr int KC_MAX = 2048;            // K chunk of a down item
constexpr int KCL = BK;                 // narrowest h chunk of an expert-local unit (one down k-tile)
constexpr int KCL_MAX = 4 * KCL;        // widest
constexpr int A_BYTES = WM * KB;        // 16 KB
constexpr int B_BYTES = LF_MAXT * KB;   // 2 KB: a 16-row h tile
constexpr int SFA_BYTES = 4 * 512;      // 4 scale atoms (one per 64 elements of K)
constexpr int SFB_BYTES = 4 * 512;
constexpr int MAX_STAGES = 10;
constexpr int HQ = 16;                  // handoff ring of down stages, weight producer -> h producer
constexpr int MIN_STAGES = 4;
constexpr int TRS = 17;                 // transpose tile row stride (floats)
constexpr int TR_FLOATS = LF_MAXT * TRS;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t SFA_COL = NACC * LF_MAXT;  // 128
constexpr uint32_t SFB_COL = SFA_COL + 16;
constexpr uint32_t XSF_COL = SFB_COL + 16;    // x scales: H/32 columns (two 64-element steps per 4)
                                              // then the two local h chunks' scales, 8 columns each
constexpr uint32_t kDevTimeout = NVFP4MOE_DEV_TIMEOUT;
constexpr int SMEM_LIMIT = 232448;

__host__ __device__ inline int lf_kc(int I) { return I < KC_MAX ? I : KC_MAX; }

// TMEM columns: accumulators, weight and h scales, x scales, then the local h chunks' scales
// (two buffers, kcl / 32 columns each) for chunks of at most kcl columns.
__host__ __device__ inline uint32_t lf_tmem_need(int H, int kcl = KCL) { return XSF_COL + uint32_t(H / 32 + kcl / 16); }

// The expert-local schedule: unit = (active expert, kcl columns of h).  One CTA runs a unit's
// kcl / 64 gate/up tiles, keeps the requantised h chunk in shared memory and runs the unit's
// down tiles (all H rows of W2, K = the chunk) from it, so no h crosses CTAs and nothing waits
// for another CTA until the combine.  Every unit is the same amount of weight bytes, so units
// go round-robin.  The chunk width kcl is the widest of 1024, 512, 256 that divides I, fits the
// h buffers (two in the stage ring's B region, whose `stages` 2 KB slots hold kcl / 128) and
// TMEM, and whose units fill the grid's rounds to at least 80 %.  Wider is better where it
// balances: a W2 row whose chunks go to different CTAs is read piecewise at different times,
// and the down stream then runs at about half the rate.  Forced (schedule 2): the widest
// balanced width, else 256; schedule 1 forces the tile-level schedule.  Returns kcl, or 0 when
// the schedule is not taken.
__host__ __device__ inline int lf_local_width(int A, int I, int G, int schedule, int H, int stages) {
  if (schedule == 1 || A < 1) return 0;
  int fallback = 0;
  for (int kcl = KCL_MAX; kcl >= KCL; kcl >>= 1) {
    if (I % kcl != 0 || I / kcl > 63 || kcl / 128 > stages || lf_tmem_need(H, kcl) > 512u) continue;
    const int64_t U = int64_t(A) * (I / kcl), rounds = (U + G - 1) / G;
    if (rounds * G * 4 <= U * 5) return kcl;
    if (kcl == KCL) fallback = kcl;
  }
  return schedule == 2 ? fallback : 0;
}

// Shapes that size the shared-memory layout: E experts, P = T*k pairs, at most AM active experts,
// at most IC work items per CTA, `stages` weight stages.
struct LfShape {
  int H, E, P, AM, IC, stages;
};

struct Layout {
  int a, x, b, sfa, sfb, xsf, tr, scl, ids, w, mask, offa, act, amask, aoff, prank, red, wsum, item, bars, total;
};

// Byte offsets of the shared-memory regions from the 1024-byte aligned base.  Operand tiles (A,
// x, B) stay 1024-byte aligned for the 128-byte swizzle; the per-slot scales 16-byte aligned.
__host__ __device__ inline Layout lf_layout(const LfShape& f) {
  Layout L;
  const int ktiles = f.H / BK;
  L.a = 0;
  L.x = L.a + f.stages * A_BYTES;
  L.b = L.x + ktiles * B_BYTES;
  L.sfa = L.b + f.stages * B_BYTES;
  L.sfb = L.sfa + f.stages * SFA_BYTES;
  L.xsf = L.sfb + f.stages * SFB_BYTES;
  L.tr = L.xsf + (f.H / 128) * 512;
  L.scl = L.tr + EPI_WARPS * TR_FLOATS * 4;  // float4 per active expert: gate, up, h and down scales
  L.ids = L.scl + f.AM * 16;                 // routing: ids [P], weights [P]
  L.w = L.ids + f.P * 4;
  L.mask = L.w + f.P * 4;                    // per expert: token bit mask [E], offsets [E+1]
  L.offa = L.mask + f.E * 4;
  L.act = L.offa + (f.E + 1) * 4;            // per active expert: id, mask, first compact pair
  L.amask = L.act + f.AM * 4;
  L.aoff = L.amask + f.AM * 4;
  L.prank = L.aoff + (f.AM + 1) * 4;         // pairs by (active expert, rank) [P]
  L.red = L.prank + f.P * 4;
  L.wsum = L.red + 32 * 4;
  L.item = L.wsum + 32 * 4;                  // this CTA's work list [IC]
  L.bars = (L.item + f.IC * 4 + HQ * 8 + 7) / 8 * 8;  // the work list, then the handoff ring [HQ][2]
  L.total = L.bars + (2 * MAX_STAGES + 2 * NACC + 1 + 2 * HQ + 3) * 8 + 16;
  return L;
}

// The shape of a launch, with the most weight stages that fit (stages 0: it does not fit).
__host__ inline LfShape lf_shape(int T, int H, int I, int E, int k, int grid) {
  LfShape f;
  f.H = H;
  f.E = E;
  f.P = T * k;
  f.AM = f.P < E ? f.P : E;
  const int nkc = (I + lf_kc(I) - 1) / lf_kc(I);
  const int64_t items = int64_t(f.AM) * (2 * I / WM + int64_t(nkc) * (H / WM));
  f.IC = int((items + grid - 1) / grid);
  for (int kcl = KCL; kcl <= KCL_MAX; kcl <<= 1) {  // the expert-local schedule, at most AM active experts
    if (I % kcl != 0) continue;
    const int64_t rounds = (int64_t(f.AM) * (I / kcl) + grid - 1) / grid;
    const int64_t ic = rounds * (kcl / 64 + H / WM);
    if (ic > f.IC) f.IC = int(ic);
  }
  f.stages = 0;
  for (int st = MAX_STAGES; st >= MIN_STAGES; --st) {
    f.stages = st;
    if (1024 + lf_layout(f).total <= SMEM_LIMIT) return f;
  }
  f.stages = 0;
  return f;
}

// Work item packing: phase (bit 0), h buffer of an expert-local unit (bit 1), K chunk (bits
// 2..7), weight tile (bits 8..20), active expert slot (bits 21..31).
__device__ __forceinline__ uint32_t lf_pack(int ph, int buf, int kc, int mt, int a) {
  return uint32_t(ph) | (uint32_t(buf) << 1) | (uint32_t(kc) << 2) | (uint32_t(mt) << 8) | (uint32_t(a) << 21);
}

struct LayerArgs {
  const __nv_bfloat16* x;   // [T][H]
  const float* logits;      // [T][E]
  int T, H, I, E, k;
  int dynamic;              // 1: x scale = amax / 2688, written to *x_scale; 0: read it
  float* x_scale;
  const uint8_t* w13_codes;
  const uint8_t* w2_codes;
  const uint8_t* w13_sf;
  const uint8_t* w2_sf;
  const float* w13_scale;   // [E][2]
  const float* w2_scale;    // [E]
  const float* h_scale;     // [E]
  float* h_amax;            // nullable [E], zeroed by the reset launch
  int32_t* ids;             // [T][k]
  float* w;                 // [T][k]
  int32_t *counts, *offsets, *padded_offsets, *pair_to_row, *row_token, *row_pair, *tile_expert, *active;
  uint8_t* x_codes;         // [rows][H/2], padded expert order (inspection copy)
  uint8_t* x_sf;            // MMA layout over the padded rows
  uint8_t* h_codes;         // [rows][I/2], padded expert order
  uint8_t* h_sf;
  float* slots;             // [T*k*nkc][H]: weighted fp32 rows by (pair, K chunk); nkc of the schedule
                            // taken, at most layer_fused_chunks(I)
  int* done;                // [min(P, E) * nkc] gate/up tiles finished per (active expert, chunk)
  int* tickets;             // [T][H/32] tile-level combine tickets
  int* gbar;                // [1] CTAs arrived at the combine barrier (expert-local)
  int schedule;             // 0: chosen from the routing; 1: tile-level; 2: expert-local
  __nv_bfloat16* out;       // [T][H]
  LfShape shape;
  uint32_t* status;
};

struct LItem {
  int ph, buf, a, mt, kc;
};

__device__ __forceinline__ LItem lf_unpack(uint32_t v) {
  LItem it;
  it.ph = int(v & 1u);
  it.buf = int((v >> 1) & 1u);
  it.kc = int((v >> 2) & 63u);
  it.mt = int((v >> 8) & 8191u);
  it.a = int(v >> 21);
  return it;
}

__device__ __forceinline__ LItem lf_item(int idx, int ng, int wt_g, int wt_d, int nkc) {
  LItem it;
  if (idx < ng) {
    it.ph = 0;
    it.buf = 0;
    it.a = idx / wt_g;
    it.mt = idx - it.a * wt_g;
    it.kc = 0;
  } else {
    const int d = idx - ng, per = nkc * wt_d;
    it.ph = 1;
    it.buf = 0;
    it.a = d / per;
    const int r = d - it.a * per;
    it.kc = r / wt_d;
    it.mt = r - it.kc * wt_d;
  }
  return it;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ int ld_relaxed_gpu(const int* ptr) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// +1 with acquire-release semantics at GPU scope; returns the previous count.
__device__ __forceinline__ int atom_acq_rel_add1(int* p) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}
// +1 with release semantics at GPU scope: the writes that precede it, including the other
// lanes' writes ordered before it by a __syncwarp, are visible to whoever acquires the count.
__device__ __forceinline__ void red_release_add1(int* p) {
  asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(p) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// silu(g) * u with the fast exponential and division (h is requantised to E2M1 right after)
__device__ __forceinline__ float lf_silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Counters, tickets and the combine barrier of one call back to zero, and the h maxima when
// they are requested.
__global__ void layer_reset_kernel(int* done, int n_done, int* tickets, int n_tickets, int* gbar, float* h_amax,
                                   int E) {
  griddep_launch_dependents();
  for (int i = threadIdx.x; i < n_done; i += blockDim.x) done[i] = 0;
  for (int i = threadIdx.x; i < n_tickets; i += blockDim.x) tickets[i] = 0;
  if (threadIdx.x == 0) *gbar = 0;
  if (h_amax)
    for (int i = threadIdx.x; i < E; i += blockDim.x) h_amax[i] = 0.0f;
}

template <int PER_LANE>
__global__ void __launch_bounds__(LF_THREADS, 1)
layer_fused_kernel(const __grid_constant__ CUtensorMap tmW13, const __grid_constant__ CUtensorMap tmW2,
                   const __grid_constant__ CUtensorMap tmH, LayerArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_shared_1024(smem_raw);
  const int T = a.T, H = a.H, I = a.I, E = a.E, k = a.k, P = T * k;
  const int S = a.shape.stages;
  const Layout L = lf_layout(a.shape);
  uint8_t* sA = smem + L.a;
  uint8_t* sX = smem + L.x;
  uint8_t* sB = smem + L.b;
  uint8_t* sSFA = smem + L.sfa;
  uint8_t* sSFB = smem + L.sfb;
  uint8_t* sXSF = smem + L.xsf;
  float* s_tr = reinterpret_cast<float*>(smem + L.tr);
  float4* s_scl = reinterpret_cast<float4*>(smem + L.scl);     // [A] sg, su, sh, sc
  int32_t* s_ids = reinterpret_cast<int32_t*>(smem + L.ids);   // [P]
  float* s_w = reinterpret_cast<float*>(smem + L.w);           // [P]
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem + L.mask);  // [E] token bit masks
  uint32_t* s_offa = reinterpret_cast<uint32_t*>(smem + L.offa);  // [E+1] offset | active offset << 16
  int32_t* s_act = reinterpret_cast<int32_t*>(smem + L.act);      // [A] active slot -> expert
  uint32_t* s_amask = reinterpret_cast<uint32_t*>(smem + L.amask);  // [A] its token mask
  int32_t* s_aoff = reinterpret_cast<int32_t*>(smem + L.aoff);      // [A+1] its first compact pair
  int32_t* s_prank = reinterpret_cast<int32_t*>(smem + L.prank);    // [P] pair at (slot, rank)
  float* s_red = reinterpret_cast<float*>(smem + L.red);            // [32]
  uint32_t* s_wsum = reinterpret_cast<uint32_t*>(smem + L.wsum);    // [32]
  uint32_t* s_item = reinterpret_cast<uint32_t*>(smem + L.item);    // [n_my] this CTA's items
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + MAX_STAGES;
  uint64_t* acc_full = bars + 2 * MAX_STAGES;
  uint64_t* acc_empty = acc_full + NACC;
  uint64_t* drain = acc_empty + NACC;
  uint64_t* hq_full = drain + 1;    // [HQ] a down stage was armed: its h loads may be issued
  uint64_t* hq_empty = hq_full + HQ;  // [HQ] the h producer took the entry
  uint64_t* h_ready = hq_empty + HQ;  // [2] local schedule: a unit's h chunk is in shared memory
  uint32_t* s_hq = s_item + a.shape.IC;  // [HQ][2] entries: stage use (ring index); item | k-tile << 16
  uint64_t* x_full = h_ready + 2;     // x staged in the (still idle) weight stage ring
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(x_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ktiles = H / BK;
  const int KC = lf_kc(I), nkc = (I + KC - 1) / KC;
  const int wt_g = 2 * I / WM, wt_d = H / WM;

  // The router logits of this warp's token (T <= 16 warps) are requested first, so that their
  // latency passes during the set-up.
  float lg[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int e = lane + 32 * i;
    lg[i] = warp < T && e < E ? __ldg(a.logits + int64_t(warp) * E + e) : 0.0f;
  }

  // ---------------------------------------------------------------- set-up ----
  if (warp == 0) {  // barrier initialisation, spread over the lanes
    for (int s = lane; s < S; s += 32) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    if (lane < NACC) {
      mbar_init(&acc_full[lane], 1);
      mbar_init(&acc_empty[lane], 4 * 32);  // the four epilogue warps of an item
    }
    for (int q = lane; q < HQ; q += 32) {
      mbar_init(&hq_full[q], 1);
      mbar_init(&hq_empty[q], 1);
    }
    if (lane == 0) {
      mbar_init(drain, 1);
      mbar_init(x_full, 1);
      *abort_flag = 0;
    }
    mbar_fence_init();
    // x (bf16, T*H*2 bytes) into the stage ring, which no weight tile uses before the routing
    // is done: one bulk copy, so that the maximum and the quantisation below read shared memory
    if (lane == 0 && int64_t(T) * H * 2 <= int64_t(S) * A_BYTES) {
      mbar_arrive_expect_tx(x_full, uint32_t(T * H * 2));
      bulk_load(sA, a.x, uint32_t(T * H * 2), x_full);
    }
  }
  if (warp == 1) {
    // columns: 8 accumulators x 16, the weight and h scales, the x scales, the local h scales
    const uint32_t need = lf_tmem_need(H, KCL_MAX);
    tmem_alloc(tmem_holder, need <= 256 ? 256u : 512u);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tmW13);
      prefetch_tensormap(&tmW2);
      prefetch_tensormap(&tmH);
    }
    // the per-expert scales are read once the active experts are known: bring them into L2 now
    for (int off = lane * 128; off < E * 8; off += 32 * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(a.w13_scale) + off));
    for (int off = lane * 128; off < E * 4; off += 32 * 128) {
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(a.w2_scale) + off));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(a.h_scale) + off));
    }
  }
  for (int e = tid; e < E; e += LF_THREADS) s_mask[e] = 0u;

  // ------------------------------------------------- routing, the x maximum ----
  // x is staged in shared memory when it fits in the stage ring (decode sizes); else it is read
  // from global memory, and quantised by the epilogue warps once the weight stream has started.
  const bool xstage = int64_t(T) * H * 2 <= int64_t(S) * A_BYTES;
  if (xstage) {  // the resident token tile and its scale staging start at zero (absent tokens, pad bytes)
    for (int i = tid; i < ktiles * B_BYTES / 16; i += LF_THREADS)
      reinterpret_cast<uint4*>(sX)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = tid; i < (H / 128) * 32; i += LF_THREADS)
      reinterpret_cast<uint4*>(sXSF)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();  // the masks are zero before any routing lane marks them
  if (warp < T) {
    const int t = warp;
    int id = 0;
    float wv = 0.0f;
    warp_topk_regs<PER_LANE>(lg, E, k, &id, &wv);
    if (lane < k) {
      s_ids[t * k + lane] = id;
      s_w[t * k + lane] = wv;
      atomicOr(&s_mask[id], 1u << t);
    }
  }
  const uint4* xs = reinterpret_cast<const uint4*>(sA);  // the staged x, 16-byte chunks
  if (xstage && !mbar_wait(x_full, 0)) atomicOr(a.status, kDevTimeout);  // the copy never landed
  if (a.dynamic) {
    // the tensor scale: amax over all of x (one-shot code, so the loops stay rolled)
    float m = 0.0f;
    const int64_t chunks = int64_t(T) * H / 8;
    const uint4* xb = reinterpret_cast<const uint4*>(a.x);
#pragma unroll 1
    for (int64_t i = tid; i < chunks; i += LF_THREADS) {
      const uint4 u = xstage ? xs[i] : __ldg(xb + i);
      const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int h = 0; h < 4; ++h)
        m = fmaxf(m, fmaxf(fabsf(__uint_as_float(q[h] << 16)), fabsf(__uint_as_float(q[h] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_red[warp] = m;
  }
  __syncthreads();

  float s_t;
  if (a.dynamic) {
    float mx = 0.0f;
    for (int i = 0; i < LF_WARPS; ++i) mx = fmaxf(mx, s_red[i]);
    s_t = __fdiv_rn(mx, 2688.0f);
  } else {
    s_t = *a.x_scale;
  }
  if (xstage) {
    // x into the resident token tile: unit = one 16-element block (token t, block b) of the
    // staged rows; codes into t's row of k-tile b / 16 (128-byte swizzle), the scale byte into
    // the staging of the x scales (512-byte block b / 8, row t at t * 16, step (b / 4) % 2 at
    // byte 8 of it)
    const int bpr = H / 16;
#pragma unroll 1
    for (int u = tid; u < T * bpr; u += LF_THREADS) {
      const int t = u / bpr, b = u - t * bpr;
      const uint4 u0 = xs[2 * u], u1 = xs[2 * u + 1];
      const uint32_t q[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      float v[16];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        v[2 * h] = __uint_as_float(q[h] << 16);
        v[2 * h + 1] = __uint_as_float(q[h] & 0xFFFF0000u);
      }
      float am = 0.0f;
#pragma unroll
      for (int h = 0; h < 16; ++h) am = fmaxf(am, fabsf(v[h]));
      float inv;
      const uint32_t sf = block_scale(am, s_t, &inv);
      const int bi = b & 15;
      *reinterpret_cast<uint2*>(sX + (b >> 4) * B_BYTES + t * KB + ((((bi >> 1) ^ (t & 7)) << 4) | ((bi & 1) << 3))) =
          encode_block16(v, inv);
      sXSF[(b >> 3) * 512 + t * 16 + ((b >> 2) & 1) * 8 + (b & 3)] = static_cast<uint8_t>(sf);
    }
    // generic stores read by the tensor core, and generic reads of the ring before the weight
    // tiles land in it: both ordered by this fence and the barriers below
    fence_proxy_async_shared();
  }

  // active experts in ascending order, their token masks, compact pair offsets: thread
  // t < 256 owns experts 4t .. 4t+3; one block scan of (pairs | active << 16)
  if (tid < LF_MAXE / 4) {
    uint32_t v[4], tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 4 * tid + i;
      const uint32_t c = e < E ? uint32_t(__popc(s_mask[e])) : 0u;
      v[i] = c | (uint32_t(c > 0) << 16);
      tot += v[i];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    named_sync(2, LF_MAXE / 4);
    uint32_t run = incl - tot;
    for (int i = 0; i < warp; ++i) run += s_wsum[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 4 * tid + i;
      if (e <= E) s_offa[e] = run;
      if (e < E && (v[i] & 0xFFFFu)) {
        const int slot = int(run >> 16);
        s_act[slot] = e;
        s_amask[slot] = s_mask[e];
        s_aoff[slot] = int(run & 0xFFFFu);
      }
      run += v[i];
    }
    if (tid == LF_MAXE / 4 - 1 && E == LF_MAXE) s_offa[E] = run;
  }
  __syncthreads();
  const int A = int(s_offa[E] >> 16);
  if (tid == 0) s_aoff[A] = P;
  for (int p = tid; p < P; p += LF_THREADS) {
    const int e = s_ids[p], t = p / k;
    const uint32_t oa = s_offa[e];
    const int rank = __popc(s_mask[e] & ((1u << t) - 1u));
    s_prank[int(oa & 0xFFFFu) + rank] = p;
  }
  // (the pair ranks are read only by the epilogue, after the barrier that follows the work list)

  // this CTA's work list, decoded once here by all threads into shared memory
  const int G = int(gridDim.x);
  const int kcl = lf_local_width(A, I, G, a.schedule, H, S);  // every CTA takes the same decision
  const bool local = kcl > 0;
  const int GU = kcl / 64;                                   // gate/up tiles per local unit
  const int U = local ? A * (I / kcl) : 0;
  const int KCx = local ? kcl : KC, nkc_x = local ? I / kcl : nkc;  // K chunk of down items, chunks
  if (local && tid == 0) {  // used only after the barrier below
    mbar_init(&h_ready[0], 4 * GU);  // the four epilogue warps of each gate/up tile of a unit
    mbar_init(&h_ready[1], 4 * GU);
  }
  const int n_u = local && int(blockIdx.x) < U ? (U - int(blockIdx.x) + G - 1) / G : 0;
  int n_my;
  if (local) {
    // units b, b + G, ... of this CTA: unit n's gate/up tiles, then, after unit n + 1's gate/up
    // tiles (MMA work while the epilogue requantises unit n's h), unit n's down tiles
    const int per = GU + wt_d;
    n_my = n_u * per;
    for (int j = tid; j < n_my; j += LF_THREADS) {
      int n, r;
      bool gu;
      if (j < GU) {
        n = 0;
        gu = true;
        r = j;
      } else {
        const int jj = j - GU, blk = jj / per, rr = jj - blk * per;
        gu = blk < n_u - 1 && rr < GU;
        n = gu ? blk + 1 : blk;
        r = gu || blk == n_u - 1 ? rr : rr - GU;
      }
      const int ug = int(blockIdx.x) + n * G, sl = ug / nkc_x, c = ug - sl * nkc_x;
      s_item[j] = gu ? lf_pack(0, n & 1, c, GU * c + r, sl) : lf_pack(1, n & 1, c, r, sl);
    }
  } else {
    // gate/up items (slot, tile), then down items (slot, chunk, tile); item idx of this CTA:
    // blockIdx.x + j * gridDim.x
    const int ng = A * wt_g, ntot = ng + A * nkc * wt_d;
    n_my = int(blockIdx.x) < ntot ? (ntot - int(blockIdx.x) + G - 1) / G : 0;
    for (int j = tid; j < n_my; j += LF_THREADS) {
      const LItem u = lf_item(int(blockIdx.x) + j * G, ng, wt_g, wt_d, nkc);
      s_item[j] = lf_pack(u.ph, 0, u.kc, u.mt, u.a);
    }
  }
  // K of a down item's chunk; its last k-tile may hold 2 of the 4 64-element steps (I % 128 == 0)
  auto kc_len = [&](int c) { return local ? kcl : min(KC, I - c * KC); };
  auto ktiles_of = [&](const LItem& w) { return w.ph == 0 ? ktiles : (kc_len(w.kc) + BK - 1) / BK; };
  auto steps_of = [&](const LItem& w, int kt) { return w.ph == 0 ? 4 : min(4, (kc_len(w.kc) - kt * BK) / 64); };
  // gate/up tiles whose h columns fall in chunk c, times the four epilogue warps of an item
  auto done_target = [&](int c) { return 4 * (kc_len(c) / 64); };
  auto abort_now = [&]() {
    *abort_flag = 1;
    atomicOr(a.status, kDevTimeout);
  };

  __syncthreads();  // the work list is read by every role
  auto item_at = [&](int j) { return lf_unpack(s_item[j]); };

  if (warp == 0) {
    // ------------------------------------------------ producer: weight tiles ----
    // This thread alone claims stages (in ring order).  A down stage also needs the h rows of
    // its expert, which the h producer loads once they are ready: the stage is handed to it
    // through the HQ ring, in order, after the stage has been armed here, so the h producer
    // never touches a stage that was not claimed for it.
    if (elect_one()) {
      uint32_t it = 0, dq = 0;
      for (int j = 0; j < n_my && !*abort_flag; ++j) {
        const LItem w = item_at(j);
        const int e = s_act[w.a];
        const int kt_n = ktiles_of(w);
        const CUtensorMap* map;
        int64_t row;
        int x0;
        const uint8_t* sf;
        if (w.ph == 0) {
          map = &tmW13;
          row = int64_t(e) * 2 * I + w.mt * WM;
          x0 = 0;
          sf = a.w13_sf + int64_t(e) * 2 * I * (H / 16) + int64_t(w.mt) * (H / 64) * 512;
        } else {
          map = &tmW2;
          row = int64_t(e) * H + w.mt * WM;
          x0 = w.kc * KCx / 2;
          sf = a.w2_sf + int64_t(e) * H * (I / 16) + (int64_t(w.mt) * (I / 64) + w.kc * (KCx / 64)) * 512;
        }
        for (int kt = 0; kt < kt_n; ++kt, ++it) {
          const int s = int(it % uint32_t(S));
          // a partial k-tile still lands a whole box (zero fill past the row); its scales are
          // the atoms that exist.  Down stages of the tile-level schedule also carry the h tile
          // and its atoms (the local schedule's h is resident).
          const bool with_h = w.ph == 1 && !local;
          const uint32_t sfb = uint32_t(steps_of(w, kt)) * 512;
          const uint32_t bytes = A_BYTES + sfb + (with_h ? B_BYTES + sfb : 0u);
          if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1)) {
            abort_now();
            break;
          }
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(sA + s * A_BYTES, map, x0 + kt * KB, int32_t(row), &full[s]);
          bulk_load(sSFA + s * SFA_BYTES, sf + int64_t(kt) * 4 * 512, sfb, &full[s]);
          if (with_h) {
            const uint32_t q = dq % HQ;
            if (!mbar_wait(&hq_empty[q], ((dq / HQ) & 1) ^ 1)) {
              abort_now();
              break;
            }
            s_hq[2 * q] = it;
            s_hq[2 * q + 1] = uint32_t(j) | (uint32_t(kt) << 16);
            mbar_arrive(&hq_full[q]);  // release: the entry is visible to the waiter
            ++dq;
          }
        }
      }
      if (*abort_flag) {  // let the copies in flight land before the CTA exits
        for (uint32_t back = 0; back < uint32_t(S) && back < it; ++back) {
          const uint32_t jj = it - 1 - back;
          mbar_wait(&full[jj % S], (jj / S) & 1, 1u << 16);
        }
      }
    }
  } else {
    // warps 2..15: x into the resident token tile when it was not staged (warp 1 waits for it)
    if (warp >= EPI_FIRST) {
      const int qt = tid - 64, qn = LF_THREADS - 64;
      if (!xstage) {  // x did not fit in the stage ring: load and quantise it here
        // one unit = one token row's 64-element K step: four 16-element blocks, 32 bytes of codes
        // and one 32-bit word of block scales
        const int nsteps = H / 64;
        for (int u = qt; u < LF_MAXT * nsteps; u += qn) {
          const int t = u / nsteps, g = u - t * nsteps;
          uint2 code[4] = {make_uint2(0u, 0u), make_uint2(0u, 0u), make_uint2(0u, 0u), make_uint2(0u, 0u)};
          uint32_t sfw = 0u;
          if (t < T) {
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
              const uint4* src = reinterpret_cast<const uint4*>(a.x + int64_t(t) * H + (g * 4 + bb) * 16);
              const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
              const uint32_t q[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
              float v[16];
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) {
                v[2 * jj] = __uint_as_float(q[jj] << 16);
                v[2 * jj + 1] = __uint_as_float(q[jj] & 0xFFFF0000u);
              }
              float amax = 0.0f;
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) amax = fmaxf(amax, fabsf(v[jj]));
              float inv;
              sfw |= block_scale(amax, s_t, &inv) << (8 * bb);
              code[bb] = encode_block16(v, inv);
            }
          }
          // k-tile g / 4, bytes 32 (g % 4) .. +32 of the 128-byte row = two 16-byte chunks,
          // swizzled by row % 8
          const int kt = g >> 2, c16 = 2 * (g & 3);
          uint8_t* rowp = sX + kt * B_BYTES + t * KB;
          *reinterpret_cast<uint4*>(rowp + ((c16 ^ (t & 7)) << 4)) =
              make_uint4(code[0].x, code[0].y, code[1].x, code[1].y);
          *reinterpret_cast<uint4*>(rowp + (((c16 + 1) ^ (t & 7)) << 4)) =
              make_uint4(code[2].x, code[2].y, code[3].x, code[3].y);
          // x scales for TMEM: 512-byte block g / 2 holds row t's scales of steps g (bytes 0..3)
          // and g + 1 (bytes 8..11) at t * 16; its copy puts them at columns +0 and +2
          uint32_t* sfp = reinterpret_cast<uint32_t*>(sXSF + (g >> 1) * 512 + t * 16 + (g & 1) * 8);
          sfp[0] = sfw;
          sfp[1] = 0u;
        }
        for (int i = qt; i < (H / 128) * 64; i += qn)  // rows 16..31 of each block: unused, zero
          reinterpret_cast<uint32_t*>(sXSF + (i >> 6) * 512 + 256)[i & 63] = 0u;
      }
      if (local)  // the local h chunks' scale staging (two 1 KB blocks, x's packing): the bytes
                  // the epilogue never writes stay zero
        for (int i = qt; i < 2 * (kcl / 128) * 128; i += qn) reinterpret_cast<uint32_t*>(sSFB)[i] = 0u;
      fence_proxy_async_shared();  // generic stores above, read by the tensor core
      // per active expert: the gate/up product scales (x scale times the weight scales), the
      // requantisation scale of h, and the down product's scale.  Only the epilogue reads them,
      // so they are loaded here, while the weight stream starts.
      for (int sl = qt; sl < A; sl += qn) {
        const int e = s_act[sl];
        const float sh = a.h_scale[e];
        s_scl[sl] = make_float4(s_t * a.w13_scale[2 * e], s_t * a.w13_scale[2 * e + 1], sh, sh * a.w2_scale[e]);
      }
    }
    named_sync(1, LF_THREADS - 32);
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 1) {
      // -------------------------------------------------------------- MMA ----
      tc_fence_after();
      if (elect_one()) {
        for (int p = 0; p < H / 128; ++p) tc_cp_sf(tmem + XSF_COL + 4 * p, desc_sf_atom(sXSF + p * 512));
        const uint32_t idesc = idesc_mxf4nvf4(WM, LF_MAXT);
        const uint32_t hsf_col = XSF_COL + uint32_t(H / 32);  // local h chunk scales, 8 columns per buffer
        uint32_t it = 0, h_par = 0u;  // bit b: the phase of h_ready[b] to wait for
        for (int j = 0; j < n_my && !*abort_flag; ++j) {
          const LItem w = item_at(j);
          const uint32_t ab = uint32_t(j) % NACC;
          if (!mbar_wait(&acc_empty[ab], ((uint32_t(j) / NACC) & 1) ^ 1)) {
            abort_now();
            break;
          }
          if (local && w.ph == 1 && w.mt == 0) {
            // a unit's first down tile: its h chunk is complete in shared memory.  Its scales
            // go to the buffer's TMEM columns; their previous reader (unit n - 2's down MMAs)
            // was issued before, and this thread's tcgen05 operations run in order.
            if (!mbar_wait(&h_ready[w.buf], (h_par >> w.buf) & 1u)) {
              abort_now();
              break;
            }
            h_par ^= 1u << w.buf;
            tc_fence_after();
            for (int p = 0; p < kcl / 128; ++p)
              tc_cp_sf(tmem + hsf_col + uint32_t(w.buf * (kcl / 32) + 4 * p),
                       desc_sf_atom(sSFB + (w.buf * (kcl / 128) + p) * 512));
          }
          tc_fence_after();
          const uint32_t d_acc = tmem + ACC_COL + ab * LF_MAXT;
          const uint32_t g0 = uint32_t((w.a * TOK_ALIGN) % 128) / 32;  // 0 or 2
          const int kt_n = ktiles_of(w);
          bool ok = true;
          for (int kt = 0; kt < kt_n; ++kt, ++it) {
            const int s = int(it % uint32_t(S));
            if (!mbar_wait(&full[s], (it / S) & 1)) {
              abort_now();
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t sfa_d = desc_sf_atom(sSFA + s * SFA_BYTES);
            const uint64_t a_d = desc_kmajor_sw128(sA + s * A_BYTES);
            if (w.ph == 0) {
#pragma unroll
              for (int q = 0; q < 4; ++q) tc_cp_sf(tmem + SFA_COL + 4 * q, sfa_d + 32 * q);
              const uint64_t b_d = desc_kmajor_sw128(sX + kt * B_BYTES);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                tc_mma_mxf4nvf4(d_acc, a_d + 2 * q, b_d + 2 * q, idesc, tmem + SFA_COL + 4 * q,
                                tmem + XSF_COL + 8 * kt + 4 * (q >> 1) + 2 * (q & 1), (kt | q) != 0 ? 1u : 0u);
            } else if (local) {
              // B = k-tile kt of the unit's resident h chunk (all 16 token rows)
              const uint64_t b_d = desc_kmajor_sw128(sB + (w.buf * (kcl / BK) + kt) * B_BYTES);
              const uint32_t hcol = hsf_col + uint32_t(w.buf * (kcl / 32) + 8 * kt);
#pragma unroll
              for (int q = 0; q < 4; ++q) tc_cp_sf(tmem + SFA_COL + 4 * q, sfa_d + 32 * q);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                tc_mma_mxf4nvf4(d_acc, a_d + 2 * q, b_d + 2 * q, idesc, tmem + SFA_COL + 4 * q,
                                tmem + hcol + 4 * (q >> 1) + 2 * (q & 1), (kt | q) != 0 ? 1u : 0u);
            } else {
              const uint64_t sfb_d = desc_sf_atom(sSFB + s * SFB_BYTES);
              const uint64_t b_d = desc_kmajor_sw128(sB + s * B_BYTES);
              const int nq = steps_of(w, kt);
              for (int q = 0; q < nq; ++q) {
                tc_cp_sf(tmem + SFA_COL + 4 * q, sfa_d + 32 * q);
                tc_cp_sf(tmem + SFB_COL + 4 * q, sfb_d + 32 * q);
              }
              for (int q = 0; q < nq; ++q)
                tc_mma_mxf4nvf4(d_acc, a_d + 2 * q, b_d + 2 * q, idesc, tmem + SFA_COL + 4 * q,
                                tmem + SFB_COL + 4 * q + g0, (kt | q) != 0 ? 1u : 0u);
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
      // counters, tickets, the combine barrier and h maxima are zeroed by the launch before this one
      griddep_wait();
      // ------------------------------------ inspection copies of the routing ----
      {
        const int64_t gt = int64_t(blockIdx.x) * (LF_THREADS - 64) + (tid - 64);
        const int64_t gs = int64_t(gridDim.x) * (LF_THREADS - 64);
        for (int64_t p = gt; p < P; p += gs) {
          const int e = s_ids[p], t = int(p) / k;
          const uint32_t oa = s_offa[e];
          const int row = int(oa >> 16) * TOK_ALIGN + __popc(s_mask[e] & ((1u << t) - 1u));
          a.ids[p] = e;
          a.w[p] = s_w[p];
          a.pair_to_row[p] = row;
          a.row_token[row] = t;
          a.row_pair[row] = int(p);
        }
        for (int64_t e = gt; e <= E; e += gs) {
          const uint32_t oa = s_offa[e];
          a.offsets[e] = int(oa & 0xFFFFu);
          a.padded_offsets[e] = int(oa >> 16) * TOK_ALIGN;
          if (e < E) a.counts[e] = __popc(s_mask[e]);
        }
        for (int64_t i = gt; i < int64_t(A) * TOK_ALIGN; i += gs) {
          const int sl = int(i / TOK_ALIGN), r = int(i % TOK_ALIGN);
          if (r == 0) {
            a.tile_expert[sl] = s_act[sl];
            a.active[1 + sl] = s_act[sl];
          }
          if (r >= __popc(s_amask[sl])) {
            a.row_token[i] = -1;
            a.row_pair[i] = -1;
          }
        }
        if (gt == 0) {
          a.active[0] = A;
          if (a.dynamic) *a.x_scale = s_t;
        }
        // x codes and scales of every pair's row (the copy of the resident tile, unswizzled)
        const int cpr = H / 32;  // 16-byte chunks per row
        for (int64_t u = gt; u < int64_t(P) * cpr; u += gs) {
          const int p = int(u / cpr), c = int(u % cpr);
          const int e = s_ids[p], t = p / k;
          const int64_t row = int64_t(s_offa[e] >> 16) * TOK_ALIGN + __popc(s_mask[e] & ((1u << t) - 1u));
          const int kt = c >> 3, c16 = c & 7;
          *reinterpret_cast<uint4*>(a.x_codes + row * (H / 2) + int64_t(c) * 16) =
              *reinterpret_cast<const uint4*>(sX + kt * B_BYTES + t * KB + ((c16 ^ (t & 7)) << 4));
        }
        for (int64_t u = gt; u < int64_t(P) * ktiles; u += gs) {
          const int p = int(u / ktiles), kt = int(u % ktiles);
          const int e = s_ids[p], t = p / k;
          const int64_t row = int64_t(s_offa[e] >> 16) * TOK_ALIGN + __popc(s_mask[e] & ((1u << t) - 1u));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int g = 4 * kt + q;
            *reinterpret_cast<uint32_t*>(a.x_sf + ((row >> 7) * (H / 64) + g) * 512 + (row & 31) * 16 +
                                         ((row & 127) >> 5) * 4) =
                *reinterpret_cast<const uint32_t*>(sXSF + (g >> 1) * 512 + t * 16 + (g & 1) * 8);
          }
        }
      }

      if (warp == HPROD_WARP && !local) {
        // ---------------------------------------------------- producer: h rows ----
        // A down item's h rows are written by the gate/up epilogues of its expert and chunk
        // (this launch); its first stage waits until their counter is complete.  The
        // counters of the next 16 items are read in one round trip and kept as a mask.  The
        // stages come from the weight producer's handoff ring, already armed for these bytes.
        if (elect_one()) {
          uint32_t ready = 0;
          int ready_base = -1;
          auto ensure_ready = [&](int j, const LItem& w) -> bool {
            if (ready_base >= 0 && j >= ready_base && j < ready_base + 16 && ((ready >> (j - ready_base)) & 1u))
              return true;
            ready_base = j;
            ready = 0;
            int v[16], tgt[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              v[i] = -1;
              tgt[i] = 0;
              if (j + i < n_my) {
                const LItem u = item_at(j + i);
                if (u.ph == 1) {
                  tgt[i] = done_target(u.kc);
                  v[i] = ld_relaxed_gpu(a.done + u.a * nkc + u.kc);
                }
              }
            }
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (v[i] >= 0 && v[i] >= tgt[i]) ready |= 1u << i;
            fence_acq_rel_gpu();
            if (!(ready & 1u)) {
              const uint64_t t0 = global_ns();
              while (ld_acquire_gpu(a.done + w.a * nkc + w.kc) < done_target(w.kc))
                if (global_ns() - t0 > 200000000ull) return false;  // 0.2 s: a gate/up tile never finished
              ready |= 1u;
            }
            return true;
          };
          // the down stages of this CTA, in the order the weight producer hands them over
          uint32_t n_down = 0;
          for (int j = 0; j < n_my; ++j) {
            const LItem w = item_at(j);
            if (w.ph == 1) n_down += uint32_t(ktiles_of(w));
          }
          bool failed = false;
          for (uint32_t dq = 0; dq < n_down; ++dq) {
            const uint32_t q = dq % HQ;
            // wait for the entry; give up if the CTA is aborting (no more entries will come)
            bool got = false;
            for (uint32_t poll = 0; poll < (1u << 22); ++poll) {
              if (mbar_try_wait(&hq_full[q], (dq / HQ) & 1)) {
                got = true;
                break;
              }
              if (*abort_flag) break;
            }
            if (!got) {
              if (!*abort_flag) abort_now();
              // aborting: the entries already handed over are armed stages; issue their loads
              // (readiness no longer matters) so that every copy of the CTA lands before it exits
              for (uint32_t dq2 = dq; dq2 < n_down; ++dq2) {
                const uint32_t q2 = dq2 % HQ;
                if (!mbar_wait(&hq_full[q2], (dq2 / HQ) & 1, 1u << 16)) break;
                const uint32_t u2 = s_hq[2 * q2], jk2 = s_hq[2 * q2 + 1];
                mbar_arrive(&hq_empty[q2]);
                const LItem w2 = item_at(int(jk2 & 0xFFFFu));
                const int kt2 = int(jk2 >> 16), s2 = int(u2 % uint32_t(S));
                const int64_t hr2 = int64_t(w2.a) * TOK_ALIGN;
                tma_load_2d(sB + s2 * B_BYTES, &tmH, w2.kc * KC / 2 + kt2 * KB, int32_t(hr2), &full[s2]);
                bulk_load(sSFB + s2 * SFB_BYTES, a.h_sf + ((hr2 >> 7) * (I / 64) + w2.kc * (KC / 64)) * 512 + int64_t(kt2) * 4 * 512,
                          uint32_t(steps_of(w2, kt2)) * 512, &full[s2]);
              }
              break;
            }
            const uint32_t st_use = s_hq[2 * q], jk = s_hq[2 * q + 1];
            mbar_arrive(&hq_empty[q]);
            const int j = int(jk & 0xFFFFu), kt = int(jk >> 16);
            const LItem w = item_at(j);
            if (kt == 0 && !failed) {
              if (!ensure_ready(j, w)) {
                abort_now();
                failed = true;  // still issue the loads of armed stages, so that they complete
              }
              fence_proxy_async_global();  // h was written through the generic proxy
            }
            const int s = int(st_use % uint32_t(S));
            const int64_t hrow = int64_t(w.a) * TOK_ALIGN;
            const uint8_t* hsf = a.h_sf + ((hrow >> 7) * (I / 64) + w.kc * (KC / 64)) * 512;
            tma_load_2d(sB + s * B_BYTES, &tmH, w.kc * KC / 2 + kt * KB, int32_t(hrow), &full[s]);
            bulk_load(sSFB + s * SFB_BYTES, hsf + int64_t(kt) * 4 * 512, uint32_t(steps_of(w, kt)) * 512, &full[s]);
          }
        }
      } else if (warp >= EPI_FIRST && warp < EPI_FIRST + EPI_WARPS) {
        // ---------------------------------------------------------- epilogue ----
        const int q = warp & 3;                    // TMEM lane quarter of this warp
        const int half = (warp - EPI_FIRST) >> 2;  // items j with j % 2 == half
        const uint32_t trow = tmem + (uint32_t(q * 32) << 16);
        float* tr = s_tr + (warp - EPI_FIRST) * TR_FLOATS;
        // a gate/up tile's h stores are counted one item later (or at the end), so that the
        // release ordering them before the count finds them drained instead of stalling
        int pending = -1;
        auto release_pending = [&]() {
          if (pending >= 0) {
            __syncwarp();
            if (lane == 0) red_release_add1(a.done + pending);
            pending = -1;
          }
        };
        for (int j = half; j < n_my && !*abort_flag; j += 2) {
          const LItem w = item_at(j);
          const uint32_t ab = uint32_t(j) % NACC;
          const int e = s_act[w.a];
          const uint32_t mask = s_amask[w.a];
          const int cnt = __popc(mask);
          const float4 scl = s_scl[w.a];
          const float sg = scl.x, su = scl.y, sh = scl.z, sc = scl.w;
          release_pending();
          if (!mbar_wait(&acc_full[ab], (uint32_t(j) / NACC) & 1)) {
            abort_now();
            break;
          }
          tc_fence_after();
          uint32_t r[16];
          tmem_ld_32x32b_x16(trow + ACC_COL + ab * LF_MAXT, r);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&acc_empty[ab]);  // the values are in registers: the accumulator is free
          if (w.ph == 0) {
            // lanes 0..15: gate rows i, lanes 16..31: up rows i of one 16-column block of h
            // (the W13 interleave); columns = tokens.  Lane l < 16 finishes tokens 0..7 of
            // column l, lane l + 16 tokens 8..15.
            const int iblk = w.mt * 4 + q;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const float send = __uint_as_float(lane < 16 ? r[8 + jj] : r[jj]);
              const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
              const float g = lane < 16 ? __uint_as_float(r[jj]) : recv;
              const float u = lane < 16 ? recv : __uint_as_float(r[8 + jj]);
              tr[(jj + 8 * (lane >> 4)) * TRS + (lane & 15)] = lf_silu_mul(g * sg, u * su);
            }
            __syncwarp();
            float amax_all = 0.0f;
            if (lane < LF_MAXT) {
              // lane t quantises token t's 16 values of this block (one block scale) if the
              // expert received token t; the other rows of a local h chunk are zero
              uint2 code = make_uint2(0u, 0u);
              uint32_t sf = 0u;
              if ((mask >> lane) & 1u) {
                float hb[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) hb[i] = tr[lane * TRS + i];
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(hb[i]));
                const int64_t row = int64_t(w.a) * TOK_ALIGN + __popc(mask & ((1u << lane) - 1u));
                float inv;
                sf = block_scale(amax, sh, &inv);
                code = encode_block16(hb, inv);
                *reinterpret_cast<uint2*>(a.h_codes + row * (I / 2) + iblk * 8) = code;
                a.h_sf[sf_mma_offset(row, iblk, I)] = static_cast<uint8_t>(sf);
                amax_all = amax;
              }
              if (local) {
                // token row `lane` of the unit's h chunk (K-major, 128-byte swizzle, k-tile
                // il / 16), and the block's scale byte in the staging the MMA warp copies to
                // TMEM (x's packing: 512-byte block il / 8, row t at t * 16, step (il / 4) % 2
                // at byte 8 of it)
                const int il = iblk - (kcl / 16) * w.kc;  // block within the chunk
                uint8_t* hrow = sB + (w.buf * (kcl / BK) + (il >> 4)) * B_BYTES + lane * KB;
                const int i16 = il & 15;
                *reinterpret_cast<uint2*>(hrow + ((((i16 >> 1) ^ (lane & 7)) << 4) | ((i16 & 1) << 3))) = code;
                sSFB[(w.buf * (kcl / 128) + (il >> 3)) * 512 + lane * 16 + ((il >> 2) & 1) * 8 + (il & 3)] =
                    uint8_t(sf);
              }
            }
            if (local) fence_proxy_async_shared();  // generic stores, read by the tensor core
            __syncwarp();
            if (local && lane == 0) mbar_arrive(&h_ready[w.buf]);
            if (a.h_amax) {
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) amax_all = fmaxf(amax_all, __shfl_xor_sync(0xffffffffu, amax_all, o));
              if (lane == 0 && amax_all > 0.0f) atomicMax(reinterpret_cast<int*>(a.h_amax + e), __float_as_int(amax_all));
            }
            if (!local) pending = w.a * nkc + (w.mt * 64) / KC;
          } else if (local) {
            // lane = output row mt*128 + 32q + lane; accumulator column = token.  The weighted
            // row of each (pair, chunk) goes to its slot; the combine follows the last unit.
            const int col = w.mt * WM + q * 32 + lane;
            const int base = s_aoff[w.a];
            for (int c = 0; c < cnt; ++c) {
              const int p = s_prank[base + c], t = p / k;
              float v = 0.0f;
#pragma unroll
              for (int i = 0; i < LF_MAXT; ++i) v = i == t ? __uint_as_float(r[i]) : v;
              a.slots[(int64_t(p) * nkc_x + w.kc) * H + col] = v * (s_w[p] * sc);
            }
          } else {
            // lane = output row mt*128 + 32q + lane; column c = the expert's c-th token; the
            // weighted row of each (pair, K chunk) goes to its slot
            const int col = w.mt * WM + q * 32 + lane;
            const int base = s_aoff[w.a];
            int my_pair = -1;
#pragma unroll
            for (int c = 0; c < LF_MAXT; ++c) {
              if (c < cnt) {
                const int p = s_prank[base + c];
                if (lane == c) my_pair = p;
                a.slots[(int64_t(p) * nkc + w.kc) * H + col] = __uint_as_float(r[c]) * (s_w[p] * sc);
              }
            }
            // one ticket per (token, 32 columns): the warp that completes a token's k x nkc
            // rows sums them in slot order and rounds once.  The ticket is an acquire-release
            // add: it publishes this warp's rows (ordered before it by the __syncwarp) and,
            // for the last one, makes the other warps' rows visible to the reads below.  (The
            // tile-level schedule spreads each token's rows over many CTAs and items, so the
            // sums are spread too; the expert-local schedule combines after a barrier instead.)
            __syncwarp();
            bool last = false;
            if (lane < cnt) last = atom_acq_rel_add1(a.tickets + (my_pair / k) * (H / 32) + (col >> 5)) == k * nkc - 1;
            uint32_t lastm = __ballot_sync(0xffffffffu, last);
            while (lastm) {
              const int c = __ffs(lastm) - 1;
              lastm &= lastm - 1;
              const int t = __shfl_sync(0xffffffffu, my_pair, c) / k;
              // the token's k x nkc rows are consecutive slot rows (pair-major, then chunk)
              const int nr = k * nkc;
              const float* rows = a.slots + int64_t(t) * nr * H + col;
              float sum = 0.0f;
              for (int r0 = 0; r0 < nr; r0 += 8) {  // up to eight loads in flight, summed in order
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = r0 + u < nr ? __ldcg(rows + int64_t(r0 + u) * H) : 0.0f;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  if (r0 + u < nr) sum += v[u];
              }
              a.out[int64_t(t) * H + col] = __float2bfloat16_rn(sum);
            }
          }
        }
        release_pending();
        // ------------------------------------------------ combine (expert-local) ----
        // Once every CTA has arrived here all slot rows are stored (one release per CTA: the
        // named barrier orders the other epilogue warps' stores before it).  Then each CTA sums
        // its slice of the [T][H] outputs over the token's k x chunks rows in slot order and
        // rounds once to bf16.  The launch is cooperative (all CTAs resident), so the wait
        // ends; it is bounded all the same.
        if (local) {
          named_sync(3, EPI_WARPS * 32);
          volatile int* s_ok = reinterpret_cast<volatile int*>(s_tr);
          float4* s_part = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(s_tr) + 4096);  // [4][64]
          if (tid == 32 * EPI_FIRST) {
            int ok = 0;
            if (!*abort_flag) {
              fence_acq_rel_gpu();
              atomicAdd(a.gbar, 1);
              const uint64_t t0 = global_ns();
              ok = 1;
              while (ld_relaxed_gpu(a.gbar) < G)
                if (global_ns() - t0 > 200000000ull) {  // 0.2 s: a CTA never arrived
                  abort_now();
                  ok = 0;
                  break;
                }
              fence_acq_rel_gpu();  // acquire, with the load that saw every arrival
            }
            *s_ok = ok;
          }
          named_sync(3, EPI_WARPS * 32);
          if (*s_ok) {
            // thread = (float4 column c4 of 64, row quarter g): quarter g sums its rows in order
            // (up to eight loads in flight), then the four partial sums are added in order
            const int nr = k * nkc_x;  // a token's slot rows are consecutive (pair-major, then chunk)
            const int64_t units = int64_t(T) * (H / 4);
            const int64_t lo = units * blockIdx.x / G, hi = units * (blockIdx.x + 1) / G;
            const int th = tid - 32 * EPI_FIRST, c4 = th & 63, g = th >> 6;
            const int rq = (nr + 3) / 4, r_lo = min(nr, g * rq), r_hi = min(nr, r_lo + rq);
            for (int64_t u0 = lo; u0 < hi; u0 += 64) {
              const int64_t u = u0 + c4;
              const int t = int(u / (H / 4)), col4 = int(u - int64_t(t) * (H / 4));
              float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              if (u < hi) {
                const float4* rows = reinterpret_cast<const float4*>(a.slots + int64_t(t) * nr * H) + col4;
                for (int r = r_lo; r < r_hi; r += 8) {
                  float4 v[8];
#pragma unroll
                  for (int q2 = 0; q2 < 8; ++q2)
                    v[q2] = r + q2 < r_hi ? __ldcg(rows + int64_t(r + q2) * (H / 4)) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
                  for (int q2 = 0; q2 < 8; ++q2)
                    if (r + q2 < r_hi) {
                      acc.x += v[q2].x;
                      acc.y += v[q2].y;
                      acc.z += v[q2].z;
                      acc.w += v[q2].w;
                    }
                }
              }
              s_part[g * 64 + c4] = acc;
              named_sync(3, EPI_WARPS * 32);
              if (g == 0 && u < hi) {
                float4 sum = s_part[c4];
#pragma unroll
                for (int q2 = 1; q2 < 4; ++q2) {
                  const float4 v = s_part[q2 * 64 + c4];
                  sum.x += v.x;
                  sum.y += v.y;
                  sum.z += v.z;
                  sum.w += v.w;
                }
                const __nv_bfloat162 lo2 = __floats2bfloat162_rn(sum.x, sum.y), hi2 = __floats2bfloat162_rn(sum.z, sum.w);
                uint2 packed;
                packed.x = *reinterpret_cast<const uint32_t*>(&lo2);
                packed.y = *reinterpret_cast<const uint32_t*>(&hi2);
                *reinterpret_cast<uint2*>(a.out + int64_t(t) * H + 4 * col4) = packed;
              }
              named_sync(3, EPI_WARPS * 32);  // s_part is rewritten next round
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    const uint32_t need = lf_tmem_need(H, KCL_MAX);
    tmem_dealloc(*tmem_holder, need <= 256 ? 256u : 512u);
  }
}

}  // namespace

bool layer_fused_fits(int T, int H, int I, int E, int k) {
  if (T < 1 || T > LF_MAXT || E < 1 || E > LF_MAXE || k < 1 || k > 32 || k > E) return false;
  if (H % BK != 0 || I % 128 != 0) return false;
  if (lf_tmem_need(H) > 512u) return false;  // the narrowest local chunk's columns too
  if (int64_t(T) * k > LF_MAXP) return false;
  const int nkc = (I + lf_kc(I) - 1) / lf_kc(I);
  if (nkc > 63 || 2 * I / WM > 8191 || H / WM > 8191) return false;  // work item packing
  return lf_shape(T, H, I, E, k, num_sms()).stages >= MIN_STAGES;
}

bool layer_fused_local_fits(int I) { return I % KCL == 0 && I / KCL <= 63; }  // width 256 at least

// Whether the expert-local schedule would be taken for the expected number of active experts
// of uniformly random routing, E * (1 - (1 - k/E)^T).
bool layer_fused_local_likely(int T, int H, int I, int E, int k) {
  if (!layer_fused_fits(T, H, I, E, k)) return false;
  const double miss = std::pow(1.0 - double(k) / E, double(T));
  const int A = int(std::lround(E * (1.0 - miss)));
  return lf_local_width(A, I, num_sms(), 0, H, lf_shape(T, H, I, E, k, num_sms()).stages) > 0;
}

// slot rows per pair: K chunks of the tile-level schedule, or of the expert-local one
int layer_fused_chunks(int I) {
  const int tile_level = (I + lf_kc(I) - 1) / lf_kc(I);
  return I % KCL == 0 && I / KCL > tile_level ? I / KCL : tile_level;
}

nvfp4moe_status launch_layer_fused_reset(const LayerFusedArgs& f, cudaStream_t s) {
  if (!layer_fused_fits(f.T, f.H, f.I, f.E, f.k))
    return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "fused layer: T=%d H=%d I=%d E=%d k=%d out of range", f.T, f.H, f.I, f.E,
                f.k);
  const int P = f.T * f.k;
  const int n_done = (P < f.E ? P : f.E) * layer_fused_chunks(f.I);
  layer_reset_kernel<<<1, 512, 0, s>>>(f.done, n_done, f.tickets, f.T * (f.H / 32), f.gbar, f.h_amax, f.E);
  return check_launch("fused layer reset");
}

nvfp4moe_status launch_layer_fused(const LayerFusedArgs& f, cudaStream_t s) {
  uint32_t* status = device_status_ptr();
  if (!status) return fail(NVFP4MOE_CUDA_ERROR, "device status word unavailable");
  if (!layer_fused_fits(f.T, f.H, f.I, f.E, f.k))
    return fail(NVFP4MOE_UNSUPPORTED_SHAPE, "fused layer: T=%d H=%d I=%d E=%d k=%d out of range", f.T, f.H, f.I, f.E,
                f.k);
  nvfp4moe_status st = NVFP4MOE_OK;
  CUtensorMap mw13, mw2, mh;
  st = make_code_map(&mw13, f.w13_codes, int64_t(f.E) * 2 * f.I, f.H, WM);
  if (st == NVFP4MOE_OK) st = make_code_map(&mw2, f.w2_codes, int64_t(f.E) * f.H, f.I, WM);
  if (st == NVFP4MOE_OK) st = make_code_map(&mh, f.h_codes, f.rows_cap, f.I, LF_MAXT);
  if (st != NVFP4MOE_OK) return st;

  LayerArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(f.x);
  a.logits = f.logits;
  a.T = f.T; a.H = f.H; a.I = f.I; a.E = f.E; a.k = f.k;
  a.dynamic = f.dynamic;
  a.x_scale = f.x_scale;
  a.w13_codes = f.w13_codes; a.w2_codes = f.w2_codes;
  a.w13_sf = f.w13_sf; a.w2_sf = f.w2_sf;
  a.w13_scale = f.w13_scale; a.w2_scale = f.w2_scale;
  a.h_scale = f.h_scale; a.h_amax = f.h_amax;
  a.ids = f.ids; a.w = f.w;
  a.counts = f.counts; a.offsets = f.offsets; a.padded_offsets = f.padded_offsets; a.pair_to_row = f.pair_to_row;
  a.row_token = f.row_token; a.row_pair = f.row_pair; a.tile_expert = f.tile_expert; a.active = f.active;
  a.x_codes = f.x_codes; a.x_sf = f.x_sf; a.h_codes = f.h_codes; a.h_sf = f.h_sf;
  a.slots = f.slots; a.done = f.done; a.tickets = f.tickets; a.gbar = f.gbar;
  a.schedule = f.schedule;
  a.out = static_cast<__nv_bfloat16*>(f.out);
  a.shape = lf_shape(f.T, f.H, f.I, f.E, f.k, num_sms());
  a.status = status;
  const int smem = 1024 + lf_layout(a.shape).total;
  const int per = (f.E + 31) / 32;
  auto go = [&](auto kern) -> cudaError_t {
    return launch_cooperative_dependent(kern, dim3(num_sms()), dim3(LF_THREADS), size_t(smem), s, mw13, mw2, mh, a);
  };
  cudaError_t e;
  if (per <= 4) {
    e = set_smem_limit_once<layer_fused_kernel<4>>(SMEM_LIMIT);
    if (e == cudaSuccess) e = go(layer_fused_kernel<4>);
  } else if (per <= 16) {
    e = set_smem_limit_once<layer_fused_kernel<16>>(SMEM_LIMIT);
    if (e == cudaSuccess) e = go(layer_fused_kernel<16>);
  } else {
    e = set_smem_limit_once<layer_fused_kernel<32>>(SMEM_LIMIT);
    if (e == cudaSuccess) e = go(layer_fused_kernel<32>);
  }
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "fused layer: %s", cudaGetErrorString(e));
  return check_launch("fused layer");
}

}  // namespace nvfp4moe
