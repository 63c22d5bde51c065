// Requantisation of h with the dynamic per-expert scale: the gate/up GEMM wrote h in fp32 and
// the amax of each expert's h over the call; here every row of padded expert order that holds
// a (token, expert) pair is quantised once that amax is known, with s_h[e] = amax_e / 2688 and
// the same block quantiser (E4M3 block scales, E2M1 codes, MMA scale layout) as the gate/up
// epilogue uses for a given scale.  The tensor scale maps the amax onto the largest E2M1
// value times the largest E4M3 block scale, 6 x 448 = 2688, as for the layer input (the
// two-level NVFP4 scaling of the Qwen3.8-Flash-Next-NVFP4-SSD-Stream model card, "What this
// model is", read as a dynamic per-tensor scale).
#include "ffn_gemm.cuh"

namespace nvfp4moe {
namespace {

__global__ void requant_h_kernel(const float* __restrict__ h_f32, int64_t rows_cap, int I, int E,
                                 const int32_t* __restrict__ padded_offsets, const int32_t* __restrict__ row_pair,
                                 const int32_t* __restrict__ tile_expert, int m_tile_log2,
                                 const float* __restrict__ h_amax, float* h_amax_user, float* h_scale,
                                 uint8_t* __restrict__ h_codes, uint8_t* __restrict__ h_sf) {
  griddep_wait();  // h and its maxima come from the gate/up GEMM launched just before
  griddep_launch_dependents();
  const int64_t gtid = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  const int64_t nthreads = int64_t(gridDim.x) * blockDim.x;
  for (int64_t e = gtid; e < E; e += nthreads) {
    // an expert without tokens keeps the neutral scale 1
    h_scale[e] = padded_offsets[e + 1] > padded_offsets[e] ? __fdiv_rn(h_amax[e], 2688.0f) : 1.0f;
    if (h_amax_user) h_amax_user[e] = h_amax[e];
  }
  const int64_t rows = padded_offsets[E] < rows_cap ? padded_offsets[E] : rows_cap;
  const int groups = I / 64;
  for (int64_t item = gtid; item < rows * groups; item += nthreads) {
    const int64_t r = item / groups;
    const int g = int(item - r * groups);
    if (row_pair[r] < 0) continue;  // a padding row
    const int e = tile_expert[r >> m_tile_log2];
    const float s_h = __fdiv_rn(h_amax[e], 2688.0f);
    const float4* src = reinterpret_cast<const float4*>(h_f32 + r * I + g * 64);
    float4 q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = src[i];
    uint2 code[4];
    uint32_t sfword = 0;
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      float v[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[4 * i] = q[4 * blk + i].x;
        v[4 * i + 1] = q[4 * blk + i].y;
        v[4 * i + 2] = q[4 * blk + i].z;
        v[4 * i + 3] = q[4 * blk + i].w;
      }
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
      float inv;
      sfword |= block_scale(amax, s_h, &inv) << (8 * blk);
      code[blk] = encode_block16(v, inv);
    }
    uint4* dst = reinterpret_cast<uint4*>(h_codes + r * (I / 2) + g * 32);
    dst[0] = make_uint4(code[0].x, code[0].y, code[1].x, code[1].y);
    dst[1] = make_uint4(code[2].x, code[2].y, code[3].x, code[3].y);
    *reinterpret_cast<uint32_t*>(h_sf + sf_mma_offset(r, 4 * g, I)) = sfword;
  }
}

}  // namespace

nvfp4moe_status launch_requant_h(const float* h_f32, int64_t rows_cap, int I, int E, const int32_t* padded_offsets,
                                 const int32_t* row_pair, const int32_t* tile_expert, int m_tile_log2,
                                 const float* h_amax, float* h_amax_user, float* h_scale, uint8_t* h_codes,
                                 uint8_t* h_sf, cudaStream_t s) {
  const int64_t items = rows_cap * (I / 64);
  int64_t blocks = (items + 255) / 256;
  if (blocks > int64_t(num_sms()) * 8) blocks = int64_t(num_sms()) * 8;
  if (blocks < 1) blocks = 1;
  const cudaError_t e = launch_dependent(requant_h_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, h_f32,
                                         rows_cap, I, E, padded_offsets, row_pair, tile_expert, m_tile_log2, h_amax,
                                         h_amax_user, h_scale, h_codes, h_sf);
  if (e != cudaSuccess) return fail(NVFP4MOE_CUDA_ERROR, "requantise h: %s", cudaGetErrorString(e));
  return check_launch("requantise h");
}

}  // namespace nvfp4moe
