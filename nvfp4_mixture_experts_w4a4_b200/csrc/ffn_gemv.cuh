// Launch interface of the decode (GEMV) kernels.
#pragma once

#include "common.cuh"

namespace nvfp4moe {

struct GemvGateUpArgs {
  int H, I;
  const uint8_t* x_codes;   // [T][H/2], token-major
  const uint8_t* x_sf;      // MMA layout over T rows
  const float* x_scale;     // [1]
  const int32_t* offsets;   // [E+1] rows of each expert (unpadded permutation)
  const int32_t* row_token; // [P]
  const int32_t* active;    // [E+1]
  const uint8_t* w13_codes;
  const uint8_t* w13_sf;
  const float* w13_scale;   // [E][2]
  const float* h_scale;     // [E]
  float* h_amax;            // nullable [E]
  uint8_t* h_codes;         // [P][I/2]
  uint8_t* h_sf;            // MMA layout over P rows
};

struct GemvDownArgs {
  int H, I;
  int ksplit;
  const uint8_t* h_codes;
  const uint8_t* h_sf;
  const int32_t* offsets;
  const int32_t* row_pair;  // [P] permuted row -> pair
  const int32_t* active;
  const uint8_t* w2_codes;
  const uint8_t* w2_sf;
  const float* w2_scale;    // [E]
  const float* h_scale;     // [E]
  const float* topk_w;      // [P] by pair; nullable (weight 1)
  float* slots;             // [ksplit][P][H]
  int64_t slot_stride;      // P*H
};

// Weight-only (W4A16) expert products for the layer's GEMV path, with the weights streamed by
// the copy engine through shared memory (stream_gemv.cu).  epi 0: gate/up (act = x [T][H] bf16
// by token, writes h_out bf16 [P][I]); epi 1: down (act = h [P][I] bf16 by permuted row,
// writes weighted fp32 slot rows [P][H] by pair).  Needs 2I % 128 == 0 and H % 128 == 0.
struct StreamA16Args {
  int H, I, E;
  const uint16_t* act;
  const int32_t* offsets;    // [E+1] unpadded permutation
  const int32_t* row_token;  // [P]
  const int32_t* row_pair;   // [P]
  const int32_t* active;     // [E+1]
  const uint8_t* w_codes;    // W13 [E][2I][H/2] or W2 [E][H][I/2]
  const uint8_t* w_sf;       // MMA layout per expert
  const float* w_scale;      // W13: [E][2]; W2: [E]
  const float* topk_w;       // [P] by pair (down)
  uint16_t* h_out;           // gate/up output
  float* slots;              // down output
  // the shared expert (bf16 weights, no scales; E = 1): shared_T > 0 tokens taken in order
  // (act rows 0..T-1, h_out [T][I], slots = its fp32 output rows [T][H], unweighted)
  int wbf16;
  int shared_T;
};
nvfp4moe_status launch_stream_gemv_a16(int epi, const StreamA16Args& a, int64_t max_active, cudaStream_t s);

// The shared expert's GEMMs on the tensor cores (tcgen05 kind::f16, dense_bf16.cu), for larger
// batches: epi 0 writes h bf16 [T][NW/2] from the interleaved W13 bf16 [NW][K] and act bf16
// [T][K]; epi 1 writes fp32 rows [T][NW] from W2 bf16 [NW][K] and h.  K % 64 == 0, NW % 128 == 0.
nvfp4moe_status launch_dense_bf16(int epi, const uint16_t* weights, const uint16_t* act, int K, int NW, int T,
                                  uint16_t* h_out, float* y_out, cudaStream_t s);

int gemv_lanes_per_row(int64_t K);
int gemv_down_ksplit(int64_t max_active, int64_t H, int64_t I);
nvfp4moe_status launch_gemv_gateup(const GemvGateUpArgs& a, int64_t max_active, cudaStream_t s);
nvfp4moe_status launch_gemv_down(const GemvDownArgs& a, int64_t max_active, cudaStream_t s);
// shared (nullable, here and in the two combines below): the shared expert's fp32 rows [T][H],
// added to each output before its bf16 rounding
nvfp4moe_status launch_combine(const float* slots, int64_t slot_stride, int ksplit,
                               const int32_t* pair_to_row, int T, int H, int k, void* out,
                               cudaStream_t s, const float* shared = nullptr);

// Small-batch prologue (route + permute + quantise x) in one launch of an 8-CTA cluster;
// see prologue.cu.
bool prologue_fits(int T, int E, int k);
nvfp4moe_status launch_prologue(const void* x, const float* logits, int T, int H, int E, int k, int m_tile,
                                int dynamic, float* x_scale, int32_t* ids, float* w, int32_t* counts, int32_t* offsets,
                                int32_t* padded_offsets, int32_t* pair_to_row, int32_t* row_token, int32_t* row_pair,
                                int32_t* tile_expert, int32_t* active, float* zero_f32, int expert_order,
                                uint8_t* x_codes, uint8_t* x_sf, int4* list, int* done, int wt_gateup, int wt_down,
                                cudaStream_t s);

// Larger-batch prologue (route + permute + quantise x) over 32-token slices in three launches;
// scratch: batch_prologue_scratch_bytes(T, E) bytes, free until the down GEMM; see
// batch_prologue.cu.  stage_events (nullable) get marks 1 and 2 after its first two launches.
bool batch_prologue_fits(int T, int E, int k);
int64_t batch_prologue_scratch_bytes(int T, int E);
nvfp4moe_status launch_batch_prologue(const void* x, const float* logits, int T, int H, int E, int k, int m_tile,
                                      int dynamic, float* x_scale, int32_t* ids, float* w, int32_t* counts,
                                      int32_t* offsets, int32_t* padded_offsets, int32_t* pair_to_row,
                                      int32_t* row_token, int32_t* row_pair, int32_t* tile_expert, int32_t* active,
                                      float* zero_f32, int expert_order, uint8_t* x_codes, uint8_t* x_sf,
                                      void* scratch, float* zero_rows, void* const* stage_events, cudaStream_t s);
// out[t] = bf16(sum_j topk_w[t*k+j] * slots[pair_to_row[t*k+j]]) in slot order, over fp32 slot
// rows in padded expert order (a programmatic dependent of the down GEMM)
nvfp4moe_status launch_combine_rows(const float* slots, const int32_t* pair_to_row, const float* topk_w, int T, int H,
                                    int k, void* out, cudaStream_t s, const float* shared = nullptr);
// out[i] = bf16(acc[i]) for the accumulating combine (a programmatic dependent of the down GEMM)
nvfp4moe_status launch_accum_to_bf16(const float* acc, int64_t n, void* out, cudaStream_t s,
                                     const float* shared = nullptr);

}  // namespace nvfp4moe
