// moe_ffn_forward: the routed NVFP4 W4A4 feed-forward layer, end to end on one stream.
//
//   route -> permute -> quantise x -> gate/up (+SwiGLU+requant) -> down -> combine
//
// All intermediates live in the caller's workspace at the offsets moe_ffn_workspace_layout
// reports; group sizes stay on the device (no host synchronisation anywhere).
#include <algorithm>

#include "ffn_gemv.cuh"
#include "ffn_gemm.cuh"

namespace nvfp4moe {
namespace {

constexpr int64_t kAlign = 256;

int64_t align_up(int64_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

nvfp4moe_status check_desc(const moe_ffn_desc* d, const char* fn) {
  NVFP4_REQUIRE(d != nullptr, NVFP4MOE_INVALID_ARG, "%s: desc is NULL", fn);
  NVFP4_REQUIRE(d->T >= 0, NVFP4MOE_INVALID_ARG, "%s: T < 0", fn);
  NVFP4_REQUIRE(d->H > 0 && d->H % 256 == 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: H=%d must be a positive multiple of 256", fn, d->H);
  NVFP4_REQUIRE(d->I > 0 && d->I % 64 == 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: I=%d must be a positive multiple of 64", fn, d->I);
  NVFP4_REQUIRE(d->E >= 1 && d->E <= 1024, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: E=%d outside [1, 1024]", fn, d->E);
  NVFP4_REQUIRE(d->top_k >= 1 && d->top_k <= 32 && d->top_k <= d->E, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: top_k=%d outside [1, min(E, 32)]", fn, d->top_k);
  NVFP4_REQUIRE(int64_t(d->T) * d->top_k <= (int64_t(1) << 24), NVFP4MOE_UNSUPPORTED_SHAPE, "%s: T*top_k > 2^24", fn);
  NVFP4_REQUIRE(d->path >= NVFP4MOE_PATH_AUTO && d->path <= NVFP4MOE_PATH_GEMM, NVFP4MOE_INVALID_ARG,
                "%s: bad path %d", fn, d->path);
  NVFP4_REQUIRE(d->x_scale_mode == NVFP4MOE_SCALE_GIVEN || d->x_scale_mode == NVFP4MOE_SCALE_DYNAMIC,
                NVFP4MOE_INVALID_ARG, "%s: bad x_scale_mode", fn);
  NVFP4_REQUIRE(d->combine >= NVFP4MOE_COMBINE_AUTO && d->combine <= NVFP4MOE_COMBINE_ACCUMULATE,
                NVFP4MOE_INVALID_ARG, "%s: bad combine mode %d", fn, d->combine);
  NVFP4_REQUIRE(d->h_scale_mode == NVFP4MOE_SCALE_GIVEN || d->h_scale_mode == NVFP4MOE_SCALE_DYNAMIC,
                NVFP4MOE_INVALID_ARG, "%s: bad h_scale_mode", fn);
  NVFP4_REQUIRE(d->act_mode == NVFP4MOE_ACT_NVFP4 || d->act_mode == NVFP4MOE_ACT_BF16, NVFP4MOE_INVALID_ARG,
                "%s: bad act_mode %d", fn, d->act_mode);
  NVFP4_REQUIRE(d->act_mode != NVFP4MOE_ACT_BF16 || d->path != NVFP4MOE_PATH_GEMM, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: the weight-only layer runs the GEMV path", fn);
  NVFP4_REQUIRE(d->shared_I >= 0 && d->shared_I % 64 == 0, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: shared_I=%d must be a multiple of 64", fn, d->shared_I);
  NVFP4_REQUIRE(d->launch_mode >= NVFP4MOE_LAUNCH_AUTO && d->launch_mode <= NVFP4MOE_LAUNCH_SINGLE_LOCAL,
                NVFP4MOE_INVALID_ARG, "%s: bad launch_mode %d", fn, d->launch_mode);
  return NVFP4MOE_OK;
}

// The shared expert runs the streamed CUDA-core kernel up to this many tokens (decode) and the
// tcgen05 bf16 GEMMs above.
constexpr int kSharedStreamMaxT = 32;

int resolve_path(const moe_ffn_desc* d) {
  if (d->act_mode == NVFP4MOE_ACT_BF16) return NVFP4MOE_PATH_GEMV;
  if (d->path != NVFP4MOE_PATH_AUTO) return d->path;
  // the weight-stationary tensor-core kernel is faster than the GEMV at every measured size
  // (decode included); the GEMV serves the shapes it does not (I % 128 != 0)
  if (d->I % 128 != 0) return NVFP4MOE_PATH_GEMV;
  return gemm_path_available() ? NVFP4MOE_PATH_GEMM : NVFP4MOE_PATH_GEMV;
}

// Batches the single-launch layer supports: at most 16 tokens on the tensor-core path with the
// ordered combine (AUTO included), given h scales and no shared expert.
bool single_launch_fits(const moe_ffn_desc* d, int path) {
  return path == NVFP4MOE_PATH_GEMM && d->act_mode == NVFP4MOE_ACT_NVFP4 && d->h_scale_mode == NVFP4MOE_SCALE_GIVEN &&
         d->shared_I == 0 && d->combine != NVFP4MOE_COMBINE_ACCUMULATE &&
         layer_fused_fits(d->T, d->H, d->I, d->E, d->top_k) &&
         (d->launch_mode != NVFP4MOE_LAUNCH_SINGLE_LOCAL || layer_fused_local_fits(d->I));
}

bool single_launch_requested(const moe_ffn_desc* d) {
  return d->launch_mode == NVFP4MOE_LAUNCH_SINGLE || d->launch_mode == NVFP4MOE_LAUNCH_SINGLE_TILE ||
         d->launch_mode == NVFP4MOE_LAUNCH_SINGLE_LOCAL;
}

// Whether this call runs as one launch.  AUTO takes it where it measured faster than the
// multi-launch path: the dense layer (one expert), and routed batches whose expected active
// experts (uniform routing) fill the grid with expert-local units.  Where routing turns out
// too skewed for those, the launch falls back to its tile-level schedule, which is correct
// but measured slower than the multi-launch path on routed batches.
bool single_launch(const moe_ffn_desc* d, int path) {
  if (d->launch_mode == NVFP4MOE_LAUNCH_MULTI || !single_launch_fits(d, path)) return false;
  return single_launch_requested(d) || d->E == 1 ||
         layer_fused_local_likely(d->T, d->H, d->I, d->E, d->top_k);
}

// AUTO: the ordered combine (faster than accumulation at the routed benchmark sizes once the
// down GEMM stores its rows with tile stores; the single launch combines in slot order too);
// with top_k = 1 on the multi-launch path accumulation adds one term per output, so it is
// exact and deterministic too, and saves the slot round trip
int resolve_combine(const moe_ffn_desc* d, int path) {
  if (d->combine != NVFP4MOE_COMBINE_AUTO) return d->combine;
  if (single_launch(d, path)) return NVFP4MOE_COMBINE_ORDERED;
  return path == NVFP4MOE_PATH_GEMM && d->top_k == 1 ? NVFP4MOE_COMBINE_ACCUMULATE : NVFP4MOE_COMBINE_ORDERED;
}

// in the slot region: the fp32 accumulator [T][H] first when accumulating, then the batch
// prologue's scratch
int64_t prologue_scratch_offset(const moe_ffn_desc* d, int combine) {
  return combine == NVFP4MOE_COMBINE_ACCUMULATE ? align_up(int64_t(d->T) * d->H * 4) : 0;
}

int64_t max_active_experts(const moe_ffn_desc* d) {
  const int64_t P = int64_t(d->T) * d->top_k;
  return P < d->E ? P : d->E;
}

void make_layout(const moe_ffn_desc* d, moe_ffn_ws_layout* L) {
  const int path = resolve_path(d);
  const int64_t T = d->T, H = d->H, I = d->I, E = d->E, k = d->top_k, P = T * k;
  const int m_tile = path == NVFP4MOE_PATH_GEMM ? grouped_token_align() : 1;
  const int64_t rows_cap = moe_permute_rows_capacity(d->T, d->E, d->top_k, m_tile);
  int64_t o = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = o;
    o = align_up(o + (bytes > 0 ? bytes : 0));
    return at;
  };
  L->path = path;
  L->m_tile = m_tile;
  L->topk_ids = take(P * 4);
  L->topk_w = take(P * 4);
  L->counts = take(E * 4);
  L->offsets = take((E + 1) * 4);
  L->padded_offsets = take((E + 1) * 4);
  L->pair_to_row = take(P * 4);
  L->row_token = take(rows_cap * 4);
  L->row_pair = take(rows_cap * 4);
  L->tile_expert = take((rows_cap / m_tile + 1) * 4);
  L->active = take((E + 1) * 4);
  L->x_scale = take(4);
  L->amax_partials = take(static_cast<int64_t>(nvfp4_quantize_workspace_size(1, T > 0 ? T : 1, H)));
  const bool a16 = d->act_mode == NVFP4MOE_ACT_BF16;  // weight-only: no activation codes
  L->x_rows = a16 ? 0 : (path == NVFP4MOE_PATH_GEMM ? rows_cap : T);
  L->x_codes = take(L->x_rows * H / 2);
  L->x_sf = take(sf_mma_bytes(L->x_rows, H));
  L->h_rows = a16 ? 0 : (path == NVFP4MOE_PATH_GEMM ? rows_cap : P);
  L->h_codes = take(L->h_rows * I / 2);
  L->h_sf = take(sf_mma_bytes(L->h_rows, I));
  L->h_bf16 = take(a16 ? P * I * 2 : 0);
  L->shared_h = take(T * int64_t(d->shared_I) * 2);
  L->shared_y = take(d->shared_I > 0 ? T * H * 4 : 0);
  // fp32 rows of the down projection: split-K partials by pair on the GEMV path; on the
  // tensor-core path rows by pair (up to 64 tokens) or by padded expert row (above), or the
  // [T][H] accumulator of the accumulating combine (the region also holds the batch
  // prologue's slice histograms until the down GEMM)
  const int combine = resolve_combine(d, path);
  const int64_t prologue_scratch = batch_prologue_scratch_bytes(d->T, d->E);
  L->combine = combine;
  L->single_launch = single_launch(d, path) ? 1 : 0;
  if (L->single_launch)  // weighted rows by (pair, K chunk)
    L->slots = take(P * layer_fused_chunks(d->I) * H * 4);
  else if (combine == NVFP4MOE_COMBINE_ACCUMULATE)
    L->slots = take(prologue_scratch_offset(d, combine) + prologue_scratch);
  else if (path == NVFP4MOE_PATH_GEMM)  // rows by pair; above 64 tokens by padded expert row
    L->slots = take(std::max<int64_t>((prologue_fits(d->T, d->E, d->top_k) ? P : rows_cap) * H * 4, prologue_scratch));
  else
    L->slots = take(std::max<int64_t>(int64_t(gemv_down_ksplit(max_active_experts(d), H, I)) * P * H * 4,
                                      prologue_scratch));
  // the fused GEMM's work list and per-expert counters, written by the small-batch prologue
  const int64_t A = P < E ? P : E;
  if (L->single_launch)  // per (active expert, K chunk) counters, per (token, 32 columns) tickets, a barrier
    L->items = take((A * layer_fused_chunks(d->I) + T * (H / 32) + 1) * 4);
  else
    L->items = take(path == NVFP4MOE_PATH_GEMM && prologue_fits(d->T, d->E, d->top_k)
                        ? grouped_fused_list_entries(A, 2 * I / 128, H / 128) * 16 + E * 4
                        : 0);
  // dynamic h scale: fp32 h before requantisation, per-expert amax and scale
  const bool dyn_h = !a16 && d->h_scale_mode == NVFP4MOE_SCALE_DYNAMIC;
  L->h_f32 = take(dyn_h ? L->h_rows * I * 4 : 0);
  L->h_stats = take(dyn_h ? 2 * E * 4 : 0);
  L->total = o;
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

nvfp4moe_status moe_ffn_workspace_layout(const moe_ffn_desc* d, moe_ffn_ws_layout* layout) {
  nvfp4moe_status st = check_desc(d, "moe_ffn_workspace_layout");
  if (st != NVFP4MOE_OK) return st;
  NVFP4_REQUIRE(layout != nullptr, NVFP4MOE_INVALID_ARG, "moe_ffn_workspace_layout: layout is NULL");
  make_layout(d, layout);
  return NVFP4MOE_OK;
}

size_t moe_ffn_workspace_size(const moe_ffn_desc* d) {
  if (check_desc(d, "moe_ffn_workspace_size") != NVFP4MOE_OK) return 0;
  moe_ffn_ws_layout L;
  make_layout(d, &L);
  return static_cast<size_t>(L.total);
}

nvfp4moe_status moe_ffn_forward(const moe_ffn_desc* d, const void* x, const float* logits, void* out,
                                void* workspace, size_t workspace_bytes, nvfp4moe_stream_t stream) {
  const char* fn = "moe_ffn_forward";
  nvfp4moe_status st = check_desc(d, fn);
  if (st != NVFP4MOE_OK) return st;
  if (d->T == 0) return NVFP4MOE_OK;
  NVFP4_REQUIRE(x && logits && out && workspace, NVFP4MOE_INVALID_ARG, "%s: NULL pointer", fn);
  NVFP4_REQUIRE(d->w13_codes && d->w13_sf && d->w13_scale && d->w2_codes && d->w2_sf && d->w2_scale,
                NVFP4MOE_INVALID_ARG, "%s: NULL weight pointer in desc", fn);
  NVFP4_REQUIRE(d->shared_I == 0 || (d->shared_w13 && d->shared_w2 && aligned16(d->shared_w13) && aligned16(d->shared_w2)),
                NVFP4MOE_INVALID_ARG, "%s: the shared expert needs 16-byte aligned shared_w13 and shared_w2", fn);
  const bool a16 = d->act_mode == NVFP4MOE_ACT_BF16;  // weight-only: no activation scales
  NVFP4_REQUIRE(a16 || d->x_scale_mode == NVFP4MOE_SCALE_DYNAMIC || d->x_scale != nullptr, NVFP4MOE_INVALID_ARG,
                "%s: GIVEN x scale needs desc->x_scale", fn);
  NVFP4_REQUIRE(aligned16(x) && aligned16(out) && aligned16(workspace) && aligned16(d->w13_codes) &&
                    aligned16(d->w13_sf) && aligned16(d->w2_codes) && aligned16(d->w2_sf),
                NVFP4MOE_INVALID_ARG, "%s: x, out, workspace and weights must be 16-byte aligned", fn);
  moe_ffn_ws_layout L;
  make_layout(d, &L);
  NVFP4_REQUIRE(workspace_bytes >= static_cast<size_t>(L.total), NVFP4MOE_WORKSPACE_TOO_SMALL,
                "%s: workspace %zu < %lld bytes", fn, workspace_bytes, (long long)L.total);
  if (L.path == NVFP4MOE_PATH_GEMM) {
    NVFP4_REQUIRE(d->I % 128 == 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: the tensor-core path needs I %% 128 == 0 (I=%d)",
                  fn, d->I);
    NVFP4_REQUIRE(d->E <= 1024, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: E > 1024", fn);
    NVFP4_REQUIRE(gemm_path_available(), NVFP4MOE_CUDA_ERROR, "%s: the tensor-core path is unavailable", fn);
  }
  NVFP4_REQUIRE(!single_launch_requested(d) || L.single_launch, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: the single launch takes at most 16 tokens on the tensor-core path with the ordered combine, "
                "given h scales and no shared expert (and I %% 256 == 0 for the expert-local schedule)", fn);
  NVFP4_REQUIRE(L.combine != NVFP4MOE_COMBINE_ACCUMULATE || L.path == NVFP4MOE_PATH_GEMM, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: the accumulating combine needs the tensor-core path", fn);
  const bool dyn_h = !a16 && d->h_scale_mode == NVFP4MOE_SCALE_DYNAMIC;
  NVFP4_REQUIRE(!dyn_h || L.path == NVFP4MOE_PATH_GEMM, NVFP4MOE_UNSUPPORTED_SHAPE,
                "%s: the dynamic h scale needs the tensor-core path", fn);
  NVFP4_REQUIRE(a16 || dyn_h || d->h_scale != nullptr, NVFP4MOE_INVALID_ARG, "%s: GIVEN h scale needs desc->h_scale",
                fn);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto I32 = [&](int64_t off) { return reinterpret_cast<int32_t*>(ws + off); };
  auto F32 = [&](int64_t off) { return reinterpret_cast<float*>(ws + off); };
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int T = d->T, H = d->H, I = d->I, E = d->E, k = d->top_k;
  const int64_t rows_cap = moe_permute_rows_capacity(T, E, k, L.m_tile);
  nvfp4moe_status mark_st = NVFP4MOE_OK;
  auto mark = [&](int i) {
    if (d->stage_events && mark_st == NVFP4MOE_OK) {
      const cudaError_t e = record_mark(d->stage_events[i], s);
      if (e != cudaSuccess) mark_st = fail(NVFP4MOE_CUDA_ERROR, "%s: stage mark %d: %s", fn, i, cudaGetErrorString(e));
    }
  };

  const bool dyn = !a16 && d->x_scale_mode == NVFP4MOE_SCALE_DYNAMIC;
  float* xs = a16 ? nullptr : (dyn ? F32(L.x_scale) : const_cast<float*>(d->x_scale));
  uint8_t* x_codes = a16 ? nullptr : ws + L.x_codes;  // the prologues quantise x only for W4A4
  const bool fused = prologue_fits(T, E, k);
  // small batches on the tensor-core path: the prologue also writes the GEMMs' work lists
  const bool lists = fused && L.path == NVFP4MOE_PATH_GEMM;
  const int64_t n_act = max_active_experts(d);
  const int64_t list_entries = grouped_fused_list_entries(n_act, 2 * I / 128, H / 128);
  int4* list = reinterpret_cast<int4*>(ws + L.items);
  int* done = reinterpret_cast<int*>(list + list_entries);
  const bool accumulate = L.combine == NVFP4MOE_COMBINE_ACCUMULATE;
  float* accum = F32(L.slots);  // fp32 [T][H] when accumulating
  uint8_t* prologue_scratch = ws + L.slots + prologue_scratch_offset(d, L.combine);
  // dynamic h scale: per-expert amax of h over this call, then the scales derived from it
  float* h_amax_int = dyn_h ? F32(L.h_stats) : (a16 ? nullptr : d->h_amax);
  float* h_scale_dyn = dyn_h ? F32(L.h_stats) + E : nullptr;

  // the shared expert (bf16 weights, streamed like the weight-only products), run before the
  // combine, which adds its fp32 rows; nullptr when there is none
  float* shared_y = d->shared_I > 0 ? F32(L.shared_y) : nullptr;
  auto run_shared = [&]() -> nvfp4moe_status {
    if (!shared_y) return NVFP4MOE_OK;
    uint16_t* hs = reinterpret_cast<uint16_t*>(ws + L.shared_h);
    if (T > kSharedStreamMaxT) {  // larger batches: tensor-core GEMMs
      nvfp4moe_status r = launch_dense_bf16(0, d->shared_w13, static_cast<const uint16_t*>(x), H, 2 * d->shared_I, T,
                                            hs, nullptr, s);
      if (r != NVFP4MOE_OK) return r;
      return launch_dense_bf16(1, d->shared_w2, hs, d->shared_I, H, T, nullptr, shared_y, s);
    }
    StreamA16Args sa{};
    sa.H = H; sa.I = d->shared_I; sa.E = 1;
    sa.wbf16 = 1; sa.shared_T = T;
    sa.act = static_cast<const uint16_t*>(x);
    sa.w_codes = reinterpret_cast<const uint8_t*>(d->shared_w13);
    sa.h_out = reinterpret_cast<uint16_t*>(ws + L.shared_h);
    nvfp4moe_status r = launch_stream_gemv_a16(0, sa, 1, s);
    if (r != NVFP4MOE_OK) return r;
    sa.act = reinterpret_cast<const uint16_t*>(ws + L.shared_h);
    sa.w_codes = reinterpret_cast<const uint8_t*>(d->shared_w2);
    sa.slots = shared_y;
    return launch_stream_gemv_a16(1, sa, 1, s);
  };

  mark(0);
  if (L.single_launch) {
    // one reset launch, then the whole layer as one persistent launch
    LayerFusedArgs f{};
    f.x = x; f.logits = logits;
    f.T = T; f.H = H; f.I = I; f.E = E; f.k = k;
    f.dynamic = dyn ? 1 : 0; f.x_scale = xs;
    f.w13_codes = d->w13_codes; f.w13_sf = d->w13_sf; f.w2_codes = d->w2_codes; f.w2_sf = d->w2_sf;
    f.w13_scale = d->w13_scale; f.w2_scale = d->w2_scale; f.h_scale = d->h_scale; f.h_amax = d->h_amax;
    f.ids = I32(L.topk_ids); f.w = F32(L.topk_w);
    f.counts = I32(L.counts); f.offsets = I32(L.offsets); f.padded_offsets = I32(L.padded_offsets);
    f.pair_to_row = I32(L.pair_to_row); f.row_token = I32(L.row_token); f.row_pair = I32(L.row_pair);
    f.tile_expert = I32(L.tile_expert); f.active = I32(L.active);
    f.x_codes = ws + L.x_codes; f.x_sf = ws + L.x_sf; f.h_codes = ws + L.h_codes; f.h_sf = ws + L.h_sf;
    f.rows_cap = rows_cap;
    f.slots = F32(L.slots);
    f.done = I32(L.items);
    f.tickets = I32(L.items) + max_active_experts(d) * layer_fused_chunks(I);
    f.gbar = f.tickets + T * (H / 32);
    f.out = out;
    f.schedule = d->launch_mode == NVFP4MOE_LAUNCH_SINGLE_TILE    ? 1
                 : d->launch_mode == NVFP4MOE_LAUNCH_SINGLE_LOCAL ? 2
                                                                  : 0;
    st = launch_layer_fused_reset(f, s);
    if (st != NVFP4MOE_OK) return st;
    mark(1);
    mark(2);
    mark(3);
    st = launch_layer_fused(f, s);
    if (st != NVFP4MOE_OK) return st;
    mark(4);
    mark(5);
    mark(6);
    return mark_st;
  }
  if (fused) {
    // small batch: routing, permutation and x quantisation in one cluster launch
    st = launch_prologue(x, logits, T, H, E, k, L.m_tile, dyn ? 1 : 0, xs, I32(L.topk_ids), F32(L.topk_w),
                         I32(L.counts), I32(L.offsets), I32(L.padded_offsets), I32(L.pair_to_row), I32(L.row_token),
                         I32(L.row_pair), I32(L.tile_expert), I32(L.active), h_amax_int,
                         L.path == NVFP4MOE_PATH_GEMM ? 1 : 0, x_codes, ws + L.x_sf, lists ? list : nullptr,
                         lists ? done : nullptr, 2 * I / 128, H / 128, s);
    if (st != NVFP4MOE_OK) return st;
    mark(1);
    mark(2);
  } else {
    // larger batch: slices of 32 tokens; x is quantised straight into its rows
    st = launch_batch_prologue(x, logits, T, H, E, k, L.m_tile, dyn ? 1 : 0, xs, I32(L.topk_ids), F32(L.topk_w),
                               I32(L.counts), I32(L.offsets), I32(L.padded_offsets), I32(L.pair_to_row),
                               I32(L.row_token), I32(L.row_pair), I32(L.tile_expert), I32(L.active), h_amax_int,
                               L.path == NVFP4MOE_PATH_GEMM ? 1 : 0, x_codes, ws + L.x_sf, prologue_scratch,
                               accumulate ? accum : nullptr, d->stage_events, s);
    if (st != NVFP4MOE_OK) return st;
  }

  if (a16) {
    // weight-only: the expert products stream their weights through shared memory
    mark(3);
    StreamA16Args sa{};
    sa.H = H; sa.I = I; sa.E = E;
    sa.offsets = I32(L.offsets); sa.row_token = I32(L.row_token); sa.row_pair = I32(L.row_pair);
    sa.active = I32(L.active);
    sa.act = static_cast<const uint16_t*>(x);
    sa.w_codes = d->w13_codes; sa.w_sf = d->w13_sf; sa.w_scale = d->w13_scale;
    sa.h_out = reinterpret_cast<uint16_t*>(ws + L.h_bf16);
    st = launch_stream_gemv_a16(0, sa, max_active_experts(d), s);
    if (st != NVFP4MOE_OK) return st;
    mark(4);
    sa.act = reinterpret_cast<const uint16_t*>(ws + L.h_bf16);
    sa.w_codes = d->w2_codes; sa.w_sf = d->w2_sf; sa.w_scale = d->w2_scale;
    sa.topk_w = F32(L.topk_w);
    sa.slots = F32(L.slots);
    st = launch_stream_gemv_a16(1, sa, max_active_experts(d), s);
    if (st != NVFP4MOE_OK) return st;
    mark(5);
    st = run_shared();
    if (st != NVFP4MOE_OK) return st;
    st = launch_combine(F32(L.slots), int64_t(T) * k * H, 1, I32(L.pair_to_row), T, H, k, out, s, shared_y);
    if (st != NVFP4MOE_OK) return st;
    mark(6);
    return mark_st;
  }
  if (L.path == NVFP4MOE_PATH_GEMV) {
    // x quantised once per token, token-major
    mark(3);
    GemvGateUpArgs g{};
    g.H = H; g.I = I;
    g.x_codes = ws + L.x_codes; g.x_sf = ws + L.x_sf; g.x_scale = xs;
    g.offsets = I32(L.offsets); g.row_token = I32(L.row_token); g.active = I32(L.active);
    g.w13_codes = d->w13_codes; g.w13_sf = d->w13_sf; g.w13_scale = d->w13_scale;
    g.h_scale = d->h_scale; g.h_amax = d->h_amax;
    g.h_codes = ws + L.h_codes; g.h_sf = ws + L.h_sf;
    st = launch_gemv_gateup(g, max_active_experts(d), s);
    if (st != NVFP4MOE_OK) return st;
    mark(4);
    GemvDownArgs dn{};
    dn.H = H; dn.I = I;
    dn.ksplit = gemv_down_ksplit(max_active_experts(d), H, I);
    dn.h_codes = ws + L.h_codes; dn.h_sf = ws + L.h_sf;
    dn.offsets = I32(L.offsets); dn.row_pair = I32(L.row_pair); dn.active = I32(L.active);
    dn.w2_codes = d->w2_codes; dn.w2_sf = d->w2_sf; dn.w2_scale = d->w2_scale;
    dn.h_scale = d->h_scale; dn.topk_w = F32(L.topk_w);
    dn.slots = F32(L.slots); dn.slot_stride = int64_t(T) * k * H;
    st = launch_gemv_down(dn, max_active_experts(d), s);
    if (st != NVFP4MOE_OK) return st;
    mark(5);
    st = run_shared();
    if (st != NVFP4MOE_OK) return st;
    st = launch_combine(F32(L.slots), dn.slot_stride, dn.ksplit, I32(L.pair_to_row), T, H, k, out, s, shared_y);
    if (st != NVFP4MOE_OK) return st;
    mark(6);
    return mark_st;
  }

  if (accumulate && fused) {  // the batch prologue zeroes the accumulator itself
    const cudaError_t e = cudaMemsetAsync(accum, 0, size_t(T) * H * 4, s);
    NVFP4_REQUIRE(e == cudaSuccess, NVFP4MOE_CUDA_ERROR, "%s: zeroing the accumulator: %s", fn, cudaGetErrorString(e));
  }
  mark(3);
  GemmFfnArgs a;
  a.T = T; a.H = H; a.I = I; a.E = E; a.k = k;
  a.rows_cap = rows_cap;
  a.x_codes = ws + L.x_codes; a.x_sf = ws + L.x_sf; a.x_scale = xs;
  a.padded_offsets = I32(L.padded_offsets); a.counts = I32(L.counts); a.active = I32(L.active);
  a.row_token = I32(L.row_token); a.row_pair = I32(L.row_pair);
  a.w13_codes = d->w13_codes; a.w13_sf = d->w13_sf; a.w13_scale = d->w13_scale;
  a.w2_codes = d->w2_codes; a.w2_sf = d->w2_sf; a.w2_scale = d->w2_scale;
  a.h_scale = dyn_h ? h_scale_dyn : d->h_scale; a.h_amax = h_amax_int;
  a.h_codes = ws + L.h_codes; a.h_sf = ws + L.h_sf;
  a.h_f32 = dyn_h ? F32(L.h_f32) : nullptr;
  a.h_amax_user = dyn_h ? d->h_amax : nullptr;
  a.tile_expert = I32(L.tile_expert);
  a.m_tile_log2 = __builtin_ctz(unsigned(L.m_tile));
  a.topk_w = F32(L.topk_w); a.slots_f32 = ws + L.slots;
  a.stage_events = d->stage_events;
  a.list = lists ? list : nullptr;
  a.list_cap = list_entries - 1;
  a.done = lists ? done : nullptr;
  a.accum = accumulate ? accum : nullptr;
  a.slots_by_row = (!accumulate && !fused) ? 1 : 0;
  st = launch_grouped_ffn(a, s);
  if (st != NVFP4MOE_OK) return st;
  st = run_shared();
  if (st != NVFP4MOE_OK) return st;
  mark(5);
  if (accumulate)
    st = launch_accum_to_bf16(accum, int64_t(T) * H, out, s, shared_y);
  else if (a.slots_by_row)
    st = launch_combine_rows(F32(L.slots), I32(L.pair_to_row), F32(L.topk_w), T, H, k, out, s, shared_y);
  else
    st = launch_combine(F32(L.slots), int64_t(T) * k * H, 1, I32(L.pair_to_row), T, H, k, out, s, shared_y);
  if (st != NVFP4MOE_OK) return st;
  mark(6);
  return mark_st;
}

}  // extern "C"
