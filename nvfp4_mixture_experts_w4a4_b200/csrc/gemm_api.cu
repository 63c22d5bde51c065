// nvfp4_gemm: one NVFP4 x NVFP4 GEMM, D = A . B^T * a_scale * b_scale.
// M <= 16 runs the split-K warp GEMV kernels of the decode path with one "expert" whose
// rows are the rows of A (partial sums reduced in a fixed order by a second kernel); larger
// M runs the tcgen05 block-scaled MMA kernel.
#include "ffn_gemm.cuh"
#include "ffn_gemv.cuh"

namespace nvfp4moe {
namespace {

constexpr int64_t kAlign = 256;
int64_t align_up(int64_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct GemvGemmLayout {
  int64_t offsets, row_pair, active, parts, total;
  int ksplit;
};

GemvGemmLayout gemv_gemm_layout(int64_t M, int64_t N, int64_t K) {
  GemvGemmLayout L;
  L.ksplit = gemv_down_ksplit(1, N, K);
  int64_t o = 0;
  L.offsets = o; o = align_up(o + 2 * 4);
  L.row_pair = o; o = align_up(o + M * 4);
  L.active = o; o = align_up(o + 2 * 4);
  L.parts = o; o = align_up(o + int64_t(L.ksplit) * M * N * 4);
  L.total = o;
  return L;
}

__global__ void gemv_gemm_init(int32_t* offsets, int32_t* row_pair, int32_t* active, int M) {
  for (int i = threadIdx.x; i < M; i += blockDim.x) row_pair[i] = i;
  if (threadIdx.x == 0) {
    offsets[0] = 0;
    offsets[1] = M;
    active[0] = 1;
    active[1] = 0;
  }
}

__global__ void reduce_parts(const float* __restrict__ parts, int ksplit, int64_t MN, void* D, int f32) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < MN; i += int64_t(gridDim.x) * blockDim.x) {
    float acc = 0.0f;
    for (int s = 0; s < ksplit; ++s) acc += parts[s * MN + i];
    if (f32)
      static_cast<float*>(D)[i] = acc;
    else
      static_cast<__nv_bfloat16*>(D)[i] = __float2bfloat16_rn(acc);
  }
}

}  // namespace
}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" {

size_t nvfp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return static_cast<size_t>(gemv_gemm_layout(M, N, K).total);
}

nvfp4moe_status nvfp4_gemm(const uint8_t* A, const uint8_t* A_sf, const float* a_scale, const uint8_t* B,
                           const uint8_t* B_sf, const float* b_scale, int64_t M, int64_t N, int64_t K, void* D,
                           int32_t d_dtype, void* workspace, size_t workspace_bytes, nvfp4moe_stream_t stream) {
  const char* fn = "nvfp4_gemm";
  NVFP4_REQUIRE(M >= 0 && N >= 0 && K >= 0, NVFP4MOE_INVALID_ARG, "%s: negative size", fn);
  NVFP4_REQUIRE(d_dtype == NVFP4MOE_DTYPE_BF16 || d_dtype == NVFP4MOE_DTYPE_F32, NVFP4MOE_INVALID_ARG,
                "%s: bad d_dtype", fn);
  NVFP4_REQUIRE(K % 128 == 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: K=%lld must be a multiple of 128", fn, (long long)K);
  NVFP4_REQUIRE(N % 128 == 0, NVFP4MOE_UNSUPPORTED_SHAPE, "%s: N=%lld must be a multiple of 128", fn, (long long)N);
  NVFP4_REQUIRE(M <= (int64_t(1) << 24), NVFP4MOE_UNSUPPORTED_SHAPE, "%s: M too large", fn);
  if (M == 0 || N == 0) return NVFP4MOE_OK;
  NVFP4_REQUIRE(A && A_sf && a_scale && B && B_sf && b_scale && D && (workspace || M > 16), NVFP4MOE_INVALID_ARG,
                "%s: NULL pointer", fn);
  NVFP4_REQUIRE(aligned16(A) && aligned16(B) && aligned16(workspace) && aligned16(D), NVFP4MOE_INVALID_ARG,
                "%s: A, B and workspace must be 16-byte aligned", fn);
  if (M > 16) {
    NVFP4_REQUIRE(gemm_path_available(), NVFP4MOE_CUDA_ERROR, "%s: the tensor-core path is unavailable", fn);
    return launch_gemm_plain(A, A_sf, a_scale, B, B_sf, b_scale, M, N, K, D, d_dtype == NVFP4MOE_DTYPE_F32,
                             reinterpret_cast<cudaStream_t>(stream));
  }
  const GemvGemmLayout L = gemv_gemm_layout(M, N, K);
  NVFP4_REQUIRE(workspace_bytes >= size_t(L.total), NVFP4MOE_WORKSPACE_TOO_SMALL, "%s: workspace %zu < %lld",
                fn, workspace_bytes, (long long)L.total);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* row_pair = reinterpret_cast<int32_t*>(ws + L.row_pair);
  int32_t* active = reinterpret_cast<int32_t*>(ws + L.active);
  float* parts = reinterpret_cast<float*>(ws + L.parts);
  gemv_gemm_init<<<1, 256, 0, s>>>(offsets, row_pair, active, static_cast<int>(M));
  nvfp4moe_status st = check_launch(fn);
  if (st != NVFP4MOE_OK) return st;
  GemvDownArgs a{};
  a.H = static_cast<int>(N);
  a.I = static_cast<int>(K);
  a.ksplit = L.ksplit;
  a.h_codes = A; a.h_sf = A_sf;
  a.offsets = offsets; a.row_pair = row_pair; a.active = active;
  a.w2_codes = B; a.w2_sf = B_sf; a.w2_scale = b_scale; a.h_scale = a_scale;
  a.topk_w = nullptr;
  a.slots = parts; a.slot_stride = M * N;
  st = launch_gemv_down(a, 1, s);
  if (st != NVFP4MOE_OK) return st;
  int64_t blocks = (M * N + 255) / 256;
  if (blocks > int64_t(num_sms()) * 8) blocks = int64_t(num_sms()) * 8;
  reduce_parts<<<static_cast<int>(blocks), 256, 0, s>>>(parts, L.ksplit, M * N, D, d_dtype == NVFP4MOE_DTYPE_F32);
  return check_launch(fn);
}

}  // extern "C"
