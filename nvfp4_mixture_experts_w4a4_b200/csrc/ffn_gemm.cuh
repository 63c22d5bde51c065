// Launch interface of the tensor-core (tcgen05 block-scaled MMA) grouped GEMM path.
#pragma once

#include "common.cuh"

namespace nvfp4moe {

// Work list of the fused decode GEMM, written by the small-batch prologue (T <= 64, so every
// active expert is one token chunk): entry 0 = {gate/up items, down items, 0, 0}; then one entry
// {expert, weight tile, first padded row, rows} per item: the gate/up items, then the down
// items, each ordered (active expert ascending, weight tile).
int64_t grouped_fused_list_entries(int64_t active_max, int64_t wt_gateup, int64_t wt_down);

struct GemmFfnArgs {
  int T, H, I, E, k;
  int64_t rows_cap;               // padded permuted rows (m_tile = grouped_token_align())
  const uint8_t* x_codes;         // [rows_cap][H/2], padded permuted rows
  const uint8_t* x_sf;            // MMA layout over rows_cap rows
  const float* x_scale;           // [1]
  const int32_t* padded_offsets;  // [E+1]
  const int32_t* counts;          // [E]
  const int32_t* active;          // [E+1]
  const int32_t* row_token;       // [rows_cap], -1 on padding rows
  const int32_t* row_pair;        // [rows_cap], -1 on padding rows
  const uint8_t* w13_codes;
  const uint8_t* w13_sf;
  const float* w13_scale;         // [E][2]
  const uint8_t* w2_codes;
  const uint8_t* w2_sf;
  const float* w2_scale;          // [E]
  const float* h_scale;           // [E]
  float* h_amax;                  // nullable
  uint8_t* h_codes;               // [rows_cap][I/2]
  uint8_t* h_sf;                  // MMA layout over rows_cap rows
  const float* topk_w;            // [T*k] by pair
  void* slots_f32;                // [T*k][H] fp32, by pair
  void* const* stage_events;      // nullable; [4] is recorded between gate/up and down
  const int4* list;               // nullable: the fused work list and the items it can hold
  int64_t list_cap;
  int* done;                      // with list: [E] gate/up completion counters, zeroed by its writer
  float* accum;                   // nullable [T][H] fp32: the down GEMM adds its rows here (zeroed)
  int slots_by_row;               // batches above 64 tokens, ordered combine: slots_f32 is
                                  // [rows_cap][H], rows in padded expert order, unweighted
  // dynamic h scale (h_f32 non-null): gate/up writes h in fp32 and its per-expert amax into
  // h_amax (zeroed); then h is requantised with h_scale[e] = h_amax[e] / 2688, which this
  // step writes, and h_amax_user (nullable) receives the maxima
  float* h_f32;
  float* h_amax_user;
  const int32_t* tile_expert;
  int m_tile_log2;
};

// Requantises fp32 h rows (the rows of padded expert order that hold a pair) with the
// per-expert scale amax / 2688; writes the scales to h_scale and, when h_amax_user is
// non-null, copies the maxima there.  A programmatic dependent of the gate/up GEMM.
nvfp4moe_status launch_requant_h(const float* h_f32, int64_t rows_cap, int I, int E, const int32_t* padded_offsets,
                                 const int32_t* row_pair, const int32_t* tile_expert, int m_tile_log2,
                                 const float* h_amax, float* h_amax_user, float* h_scale, uint8_t* h_codes,
                                 uint8_t* h_sf, cudaStream_t s);

bool gemm_path_available();
int grouped_token_align();
// gate/up (SwiGLU + requant) then down (fp32 slot rows or accumulator), weight-stationary
// grouped GEMM
nvfp4moe_status launch_grouped_ffn(const GemmFfnArgs& a, cudaStream_t s);
// D[M][N] = A . B^T * a_scale[0] * b_scale[0]; N % 128 == 0, K % 128 == 0.
nvfp4moe_status launch_gemm_plain(const uint8_t* A, const uint8_t* A_sf, const float* a_scale, const uint8_t* B,
                                  const uint8_t* B_sf, const float* b_scale, int64_t M, int64_t N, int64_t K, void* D,
                                  int d_f32, cudaStream_t s);

// The whole layer as one persistent launch (plus a small reset launch before it) for batches
// of at most 16 tokens: routing, permutation, x quantisation, both GEMMs and the ordered
// combine.  It writes the same intermediates as the multi-launch path (padded expert order,
// m_tile = 64) and the output.
struct LayerFusedArgs {
  const void* x;
  const float* logits;
  int T, H, I, E, k;
  int dynamic;
  float* x_scale;
  const uint8_t *w13_codes, *w13_sf, *w2_codes, *w2_sf;
  const float *w13_scale, *w2_scale, *h_scale;
  float* h_amax;  // nullable
  int32_t* ids;
  float* w;
  int32_t *counts, *offsets, *padded_offsets, *pair_to_row, *row_token, *row_pair, *tile_expert, *active;
  uint8_t *x_codes, *x_sf, *h_codes, *h_sf;
  int64_t rows_cap;
  float* slots;   // [T*k*layer_fused_chunks(I)][H] fp32
  int* done;      // [min(T*k, E) * layer_fused_chunks(I)]
  int* tickets;   // [T][H/32] tile-level combine tickets
  int* gbar;      // [1] the expert-local combine barrier
  int schedule;   // 0: chosen per call from the routing; 1: tile-level; 2: expert-local
  void* out;
};
bool layer_fused_fits(int T, int H, int I, int E, int k);
int layer_fused_chunks(int I);
bool layer_fused_local_fits(int I);  // the expert-local schedule applies (I % 256 == 0)
// the expert-local schedule would be taken for uniformly random routing of this shape
bool layer_fused_local_likely(int T, int H, int I, int E, int k);
// the reset launch (counters, barrier, h maxima to zero), then the layer launch (cooperative),
// its programmatic dependent; nothing else may run on the stream between the two
nvfp4moe_status launch_layer_fused_reset(const LayerFusedArgs& f, cudaStream_t s);
nvfp4moe_status launch_layer_fused(const LayerFusedArgs& f, cudaStream_t s);

}  // namespace nvfp4moe
